// permute.cu -- the layout transformation of "Sparse VideoGen: Accelerating
// Video Diffusion Transformers with Spatial-Temporal Sparsity" (Abstract:
// "hardware-efficient tensor layout transformation"), which makes a temporal
// head's slash pattern block-banded, and its inverse (SVG2 explainer, 2.A:
// permuting before attention and back after leaves the output unchanged).
//
// Token (i, j) moves between frame-major row x = i*F + j and token-major row
// x' = j*N + i.  Every row is d contiguous elements (128 or 256 bytes in
// bf16), so the transformation is a row gather: each 16-byte chunk is read
// once and written once, and both sides touch whole rows, i.e. whole 32-byte
// sectors.  The kernel walks the DESTINATION head row by row (coalesced
// streaming stores; the rows are adjacent in [B, H, L, d] and H*d apart in
// [B, L, H, d]) and gathers source rows; a block handles one slab of one
// head of one tensor and exits at once for heads the label says stay put.
#include "internal.h"

namespace svg {
namespace {

struct PermuteParams {
  const uint4* src[3];
  uint4* dst[3];
  HeadStrides ss, ds;  // in 16-byte chunks
  const int8_t* label;
  int sel;                    // heads whose label equals sel move
  long long chunks_per_head;  // L * row_chunks
  int row_chunks;             // 16-byte chunks per row
  int BH, N, F;
  int to_token_major;
};

constexpr int kPermThreads = 256;
constexpr int kPermUnroll = 4;

__global__ void __launch_bounds__(kPermThreads) permute_rows_kernel(const __grid_constant__ PermuteParams p) {
  const int t = blockIdx.y / p.BH;       // tensor
  const int bh = blockIdx.y - t * p.BH;  // head
  if (p.label != nullptr && p.label[bh] != p.sel) return;
  const uint4* __restrict__ src = p.src[t] + p.ss.head(bh);
  uint4* __restrict__ dst = p.dst[t] + p.ds.head(bh);
  const int rc = p.row_chunks;
  const long long srs = p.ss.sl, drs = p.ds.sl;  // row strides
  const long long step = static_cast<long long>(gridDim.x) * kPermThreads * kPermUnroll;
  for (long long base = static_cast<long long>(blockIdx.x) * kPermThreads * kPermUnroll + threadIdx.x;
       base < p.chunks_per_head; base += step) {
    uint4 val[kPermUnroll];
    long long didx[kPermUnroll];
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      const long long e = base + static_cast<long long>(u) * kPermThreads;
      didx[u] = -1;
      if (e < p.chunks_per_head) {
        const int row = static_cast<int>(e / rc);
        const int c = static_cast<int>(e - static_cast<long long>(row) * rc);
        didx[u] = row * drs + c;
        int srow;
        if (p.to_token_major) {  // dst row x' = j*N + i  <-  src row i*F + j
          const int j = row / p.N, i = row - j * p.N;
          srow = i * p.F + j;
        } else {  // dst row x = i*F + j  <-  src row j*N + i
          const int i = row / p.F, j = row - i * p.F;
          srow = j * p.N + i;
        }
        val[u] = __ldg(src + srow * srs + c);
      }
    }
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u)
      if (didx[u] >= 0) __stcs(dst + didx[u], val[u]);
  }
}

}  // namespace

svg_status launch_permute(int ntensors, const void* const* src, void* const* dst, int BH, int N, int F, int d,
                          int elem_bytes, const HeadStrides& ss, const HeadStrides& ds, const int8_t* label,
                          bool to_token_major, cudaStream_t stream, int sel) {
  const int row_bytes = d * elem_bytes;
  if (row_bytes % 16 != 0) return fail(SVG_ERR_UNSUPPORTED, "row of %d bytes is not a multiple of 16", row_bytes);
  // element strides -> 16-byte chunks (every stride is a multiple of d)
  const int per = 16 / elem_bytes;
  auto chunks = [per](HeadStrides s) {
    s.sb /= per;
    s.sh /= per;
    s.sl /= per;
    return s;
  };
  PermuteParams p{};
  p.ss = chunks(ss);
  p.ds = chunks(ds);
  for (int t = 0; t < ntensors; ++t) {
    p.src[t] = static_cast<const uint4*>(src[t]);
    p.dst[t] = static_cast<uint4*>(dst[t]);
  }
  p.label = label;
  p.sel = sel;
  p.row_chunks = row_bytes / 16;
  p.chunks_per_head = static_cast<long long>(N) * F * p.row_chunks;
  p.BH = BH;
  p.N = N;
  p.F = F;
  p.to_token_major = to_token_major ? 1 : 0;
  const long long per_block = static_cast<long long>(kPermThreads) * kPermUnroll;
  long long bx = (p.chunks_per_head + per_block - 1) / per_block;
  // Enough blocks per head to fill the 148 SMs several times over across all
  // heads, but no more than the slab count.
  const long long want = (148LL * 16 + static_cast<long long>(BH) * ntensors - 1) /
                         (static_cast<long long>(BH) * ntensors);
  if (bx > want) bx = want;
  if (bx < 1) bx = 1;
  if (static_cast<long long>(BH) * ntensors > 65535)
    return fail(SVG_ERR_UNSUPPORTED, "B*H*tensors = %lld exceeds the grid limit",
                static_cast<long long>(BH) * ntensors);
  dim3 grid(static_cast<unsigned>(bx), static_cast<unsigned>(BH * ntensors));
  permute_rows_kernel<<<grid, kPermThreads, 0, stream>>>(p);
  return cuda_check(cudaGetLastError(), "permute launch");
}

}  // namespace svg
