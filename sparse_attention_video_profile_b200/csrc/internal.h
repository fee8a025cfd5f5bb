// internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "svg.h"

// Range checks of the debug build (libsvg_debug.so, -DSVG_DEBUG_BOUNDS=1).
#ifndef SVG_DEBUG_BOUNDS
#define SVG_DEBUG_BOUNDS 0
#endif

namespace svg {

// Upper bound on any single pipeline wait inside a kernel.  Waits in a
// healthy run last microseconds; the bound only turns a stall into an error.
constexpr uint64_t kDefaultWaitNs = 1000000000ull;

// Records a message for svg_last_error() and returns `st`.
svg_status fail(svg_status st, const char* fmt, ...);
// Maps a CUDA error to SVG_ERR_CUDA with a message; SVG_OK if e == cudaSuccess.
svg_status cuda_check(cudaError_t e, const char* what);

// ------------------------------------------------------------- tensor layout

// Where the rows of a q/k/v/o tensor live.  Head bh of a call (bh = b*H + h
// over the call's own heads) is head g = bh + bh0 of the tensor, whose nb
// batch entries hold H heads each; element c of row x of that head sits at
// element (g / H)*sb + (g % H)*sh + x*sl + c.  [B, H, L, d]: sb = H*L*d,
// sh = L*d, sl = d.  [B, L, H, d]: sb = L*H*d, sh = d, sl = H*d.
struct HeadStrides {
  int H, nb, bh0;
  long long sb, sh, sl;
  __host__ __device__ long long head(int bh) const {
    const int g = bh + bh0;
    return static_cast<long long>(g / H) * sb + static_cast<long long>(g % H) * sh;
  }
  // TMA coordinates (head, batch entry) of call head bh
  __host__ __device__ int tma_h(int bh) const { return (bh + bh0) % H; }
  __host__ __device__ int tma_b(int bh) const { return (bh + bh0) / H; }
};
// Contiguous [B, H, L, d] (workspace copies are always laid out this way).
HeadStrides dense_strides(int B, int H, int L, int d);
// The caller's tensors of a call on `s` (s->layout).
HeadStrides shape_strides(const svg_shape* s);

// TMA views (bf16, 128-byte swizzle) of a tensor laid out as s, indexed by
// (column, row, tma_h, tma_b):
// tiles (d, L, H, nb) with 64 x 128 x 1 x 1 boxes (attn_sm100.cu);
svg_status make_tile_map_bf16(CUtensorMap* map, const void* base, const HeadStrides& s, int L, int D);
// frame groups (d, frame, position, H, nb) of a frame-major tensor with
// `size` frames x 128/size positions per box, indexed (column, first frame,
// first position, tma_h, tma_b).
svg_status make_group_map_bf16(CUtensorMap* map, const void* base, const HeadStrides& s, int N, int F, int D,
                               int size);

// ------------------------------------------------------------- permute

// Moves rows between frame-major (x = i*F + j) and token-major (x' = j*N + i)
// order for up to three tensors.  to_token_major: src frame-major -> dst
// token-major; otherwise the inverse.  label == nullptr: every head.
// Only heads whose label equals `sel` move (SVG_TEMPORAL unless given).
// Rows of d elements of elem_bytes each; src and dst laid out as ss and ds.
svg_status launch_permute(int ntensors, const void* const* src, void* const* dst, int BH, int N, int F, int d,
                          int elem_bytes, const HeadStrides& ss, const HeadStrides& ds, const int8_t* label,
                          bool to_token_major, cudaStream_t stream, int sel = SVG_TEMPORAL);

// ------------------------------------------------------------- attention

struct BandAttnArgs {
  int B, H, L, d;
  int dtype;  // svg_dtype
  float scale;
  // Layouts: hs of q, k, v, o; hsp of qp, kp, vp, op (and, in the SVG2 mode,
  // of the cluster-permuted q, k, v).
  HeadStrides hs, hsp;
  // frame-major tensors (spatial heads, or all heads when label == nullptr)
  const void *q, *k, *v;
  void* o;
  // token-major tensors (temporal heads)
  const void *qp, *kp, *vp;
  void* op;
  const int8_t* label;  // nullptr -> every head uses band 0 on (q, k, v, o)
  int G0, a0;           // band of label-0 heads
  int G1, a1;           // band of label-1 heads
  const int8_t* modes;  // mixed-pattern modes (overrides label), or nullptr
  int win, md_a, stripe, N;
  int* status;          // device status word (never null here)
  uint64_t wait_ns;
  int withhold_loads;   // self-test of the bounded waits (tcgen05 kernel only)
  // Fused layout transformation (tcgen05 kernel only): heads that run
  // token-major read their rows straight from (q, k, v) through frame-group
  // boxes and write O rows back to frame-major positions of o; qp..op are
  // unused.  Needs N (frames) > 0.
  int fused;
  // SVG2 cluster-pair mode (tcgen05 kernel only, overrides label and modes):
  // q, k, v are the cluster-permuted tensors; query row r (permuted) is in
  // cluster s2_cid[r] and lands at row s2_perm[r] of o; it attends to the key
  // clusters its cluster keeps (bit ck of s2_sel[cq]), which occupy permuted
  // key rows [s2_koff[ck], s2_koff[ck + 1]).
  int s2, s2_Cq, s2_Ck;
  const int32_t* s2_cid;
  const int32_t* s2_perm;
  const int32_t* s2_koff;
  const uint32_t* s2_sel;
};

// SVG2 workspace pieces (bytes, 256-aligned) for B*H heads of L rows.
struct Svg2Sizes {
  int nblk, W;
  size_t hist, perm, off_q, off_k, mu_q, mu_k, tensor, total;
};
Svg2Sizes svg2_sizes(int BH, int L, int Cq, int Ck, int d);
svg_status svg2_sort(const int32_t* assign, int BH, int L, int C, int nblk, int32_t* hist, int32_t* perm,
                     int32_t* cid, int32_t* off, int* status, cudaStream_t stream);
svg_status svg2_gather(const void* src, const HeadStrides& ss, const int32_t* perm, void* dst, int BH, int L, int d,
                       cudaStream_t stream);
svg_status svg2_centroids(const void* xp, const int32_t* off, int BH, int L, int C, int d, float* mu,
                          cudaStream_t stream);
svg_status svg2_topp(const float* mu_q, const float* mu_k, const int32_t* off_k, int BH, int Cq, int Ck, int d,
                     float scale, float p, uint32_t* sel, cudaStream_t stream);
// k-means (kmeans_sm100.cu): workspace bytes and the Lloyd iterations.
size_t kmeans_workspace_bytes(int BH, int L, int C, int d);
svg_status launch_kmeans(const void* x, const HeadStrides& xs, int BH, int L, int C, int d, int iters, int32_t* assign,
                         float* mu, void* workspace, int* status, cudaStream_t stream);

svg_status launch_attn_sm100(const BandAttnArgs& a, cudaStream_t stream);
// Frame groups of the fused layout transformation: powers of two, largest
// first, at most 128 frames each.  Writes their log2 sizes to glog and
// returns how many there are, or -1 if more than max_groups are needed.
int fused_frame_groups(int N, int* glog, int max_groups);
// Key tiles (128 keys) one token-major head with positional half-width a
// (keys |j1 - j2| < a, a <= F) takes over all its query rows: with
// token-major copies (`separate`) and with the fused layout (`fused`, the
// same CTA geometry as the kernel).
void token_major_tile_counts(int N, int F, int a, long long* separate, long long* fused);
// True when the fused layout does at most 3 % more attention work than the
// token-major copies (about what the permute + unpermute passes cost).
bool fused_layout_preferred(int N, int F, int a);
// The choice svg_sparse_3d_attn makes (and its host-buffer form): bf16,
// [B, H, L, d] tensors and fused_layout_preferred with the clamped temporal
// band.
bool whole_call_fused(const svg_shape* s, int a2);
svg_status launch_attn_simt(const BandAttnArgs& a, cudaStream_t stream);
// fp32 tensors on the tensor cores in tf32 (attn_tf32.cu): bands with or
// without labels (no modes, fused layout or SVG2 mode).
svg_status launch_attn_tf32(const BandAttnArgs& a, cudaStream_t stream);
// Tile shape of the tcgen05 kernel (rows of Q per tile, keys per tile).
constexpr int kAttnBq = 128;
constexpr int kAttnBk = 128;

// ------------------------------------------------------------- profiling

struct ProfileLayout {
  int S_pad;      // sampled rows rounded up to the row-block of the kernel
  int n_chunks;   // key chunks per head
  int chunk;      // keys per chunk (multiple of 64)
  size_t o_bytes;     // partial outputs  [BH][n_chunks][3][S_pad][d] f32
  size_t ml_bytes;    // partial max/sum  [BH][n_chunks][3][S_pad][2] f32
  size_t part_bytes;  // per-row sums [BH][S_pad][3] f64: (O_1 - O_d)^2, (O_2 - O_d)^2, O_d^2
  size_t status_bytes;  // the call's own device status word (int32, zeroed by the call), padded to 256 bytes
  size_t total;         // o_bytes + ml_bytes + part_bytes + status_bytes
};

// Offset of the call's status word inside a profiling workspace.
inline size_t profile_status_offset(const ProfileLayout& lay) { return lay.o_bytes + lay.ml_bytes + lay.part_bytes; }

// Workspace layout of the profiling kernels.  max_chunks > 0 caps the number
// of key chunks (fewer chunks need less workspace); chunk_len > 0 fixes the
// keys per chunk instead of choosing them for the head count, so a call on a
// subset of heads splits the keys, and rounds, exactly as a call on all of
// them.  bf16 chunks are whole 128-key tiles, fp32 chunks (CUDA cores)
// multiples of 32 keys, at least 1024 unless the sequence is shorter.
bool profile_layout(int B, int H, int L, int d, int dtype, int S, ProfileLayout* out, int max_chunks = 0,
                    int chunk_len = 0);

// Online profiling.  Device-side failures (a wait that ran out, in-band
// weights that underflowed) are recorded in the status word inside `ws`
// (zeroed first, so calls with separate workspaces do not interfere) and,
// when status_out is not NULL, also OR-ed into *status_out.
svg_status launch_profile(int B, int H, int N, int F, int d, int dtype, float scale, const void* q,
                          const void* k, const void* v, const HeadStrides& hs, int a1, int a2, const int32_t* rows, int S,
                          float* mse, int8_t* label, void* ws, const ProfileLayout& lay,
                          int* status_out, cudaStream_t stream);

// Masks of the two restricted variants of a profiling pass.
constexpr int kProfFrameBand = 0;     // |i_x - i_y| < a           (spatial)
constexpr int kProfPositionBand = 1;  // |j_x - j_y| < a           (temporal, multi-diagonal)
constexpr int kProfWindow = 2;        // |x - y| <= a              (diagonal)
constexpr int kProfPrefix = 3;        // y < a                     (vertical stripe)
constexpr int kProfNone = 4;          // no key

// bf16 stage 1 of profiling on the tensor cores (profile_sm100.cu): dense and
// two restricted variants (kind[v], par[v]) of the sampled rows' attention.
svg_status launch_profile_sm100(int BH, int N, int F, int d, float scale, const void* q, const void* k,
                                const void* v, const HeadStrides& hs, const int (&kind)[2], const int (&par)[2], const int32_t* rows, int S,
                                float* ws_o, float* ws_ml, int nch, int chunk, int* status, cudaStream_t stream);

// One profiling pass: stage 1 with the given variants, then the per-row sums
// part[bh][s][3] = {sum (O_1 - O_d)^2, sum (O_2 - O_d)^2, sum O_d^2} over d.
svg_status launch_profile_pass(int B, int H, int N, int F, int d, int dtype, float scale, const void* q,
                               const void* k, const void* v, const HeadStrides& hs, const int (&kind)[2], const int (&par)[2],
                               const int32_t* rows, int S, void* ws, const ProfileLayout& lay, double* part,
                               int* status, cudaStream_t stream);

// Sparse-vDiT mode search: two passes (diagonal, multi-diagonal) and (stripe,
// none) plus the selection kernel.  part2 holds the second pass's sums.
svg_status launch_mode_search(int B, int H, int N, int F, int d, float scale, const void* q, const void* k,
                              const void* v, const HeadStrides& hs, const int32_t* rows, int S, int window, int md_half, int stripe,
                              float lambda, float epsilon, float* loss, int8_t* mode, void* ws,
                              const ProfileLayout& lay, double* part2, cudaStream_t stream);

// A zeroed per-device status word for kernels whose entry point takes none.
// It is shared by every such call on the device.
svg_status internal_status_word(int** out, cudaStream_t stream);

// svg_profile_heads with the failure bits also OR-ed into status_out (may be
// NULL); the whole calls use it to carry a profiling failure to the caller.
// q, k, v are laid out as hs.  chunk_len > 0 fixes the profiling key split
// (see profile_layout).
svg_status profile_heads_impl(const svg_shape* shape, const HeadStrides& hs, const void* q, const void* k,
                              const void* v, int32_t a1,
                              int32_t a2, const int32_t* rows, int32_t S, float* mse, int8_t* label, void* workspace,
                              size_t workspace_bytes, int32_t* status_out, cudaStream_t stream, int chunk_len = 0);

}  // namespace svg
