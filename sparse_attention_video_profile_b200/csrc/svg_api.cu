// svg_api.cu -- the C ABI declared in include/svg.h: argument checking,
// workspace accounting and kernel dispatch.  No entry point allocates
// memory or synchronises the stream.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "internal.h"

namespace svg {

static thread_local char g_last_error[512] = "";

svg_status fail(svg_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

svg_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return SVG_OK;
  return fail(SVG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Per-device status word used when the caller passes no status_dev.
__device__ int g_internal_status;

namespace {

size_t elem_size(int dtype) { return dtype == SVG_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

svg_status check_shape(const svg_shape* s) {
  if (s == nullptr) return fail(SVG_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 1 || s->H < 1 || s->N < 1 || s->F < 1 || s->d < 1)
    return fail(SVG_ERR_INVALID_ARG, "B, H, N, F, d must be >= 1 (got %d %d %d %d %d)", s->B, s->H, s->N, s->F, s->d);
  if (static_cast<long long>(s->N) * s->F > (1LL << 30))
    return fail(SVG_ERR_INVALID_ARG, "L = N*F = %lld is too large", static_cast<long long>(s->N) * s->F);
  if (s->dtype != SVG_BF16 && s->dtype != SVG_FP32 && s->dtype != SVG_TF32)
    return fail(SVG_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
  if (s->layout != SVG_LAYOUT_BHLD && s->layout != SVG_LAYOUT_BLHD)
    return fail(SVG_ERR_INVALID_ARG, "unknown layout %d", s->layout);
  if (!(s->scale >= 0.f) || isinf(s->scale)) return fail(SVG_ERR_INVALID_ARG, "scale must be finite and >= 0");
  if (s->dtype == SVG_BF16 && s->d != 64 && s->d != 128)
    return fail(SVG_ERR_UNSUPPORTED, "bf16 supports d in {64, 128}, got %d", s->d);
  if (s->dtype != SVG_BF16 && s->d != 32 && s->d != 64 && s->d != 128)
    return fail(SVG_ERR_UNSUPPORTED, "fp32 / tf32 support d in {32, 64, 128}, got %d", s->d);
  return SVG_OK;
}

float eff_scale(const svg_shape* s) { return s->scale > 0.f ? s->scale : 1.0f / sqrtf(static_cast<float>(s->d)); }

svg_status check_tensors(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(SVG_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (!aligned16(p)) return fail(SVG_ERR_INVALID_ARG, "a tensor pointer is not 16-byte aligned");
  }
  return SVG_OK;
}

// Clamp a band so that (g + a) * G cannot overflow: a >= ceil(L/G) already
// keeps every pair.
int clamp_band(int a, int G, int L) {
  const int full = (L + G - 1) / G;
  return a > full ? full : a;
}

}  // namespace

HeadStrides dense_strides(int B, int H, int L, int d) {
  HeadStrides s;
  s.H = H;
  s.nb = B;
  s.bh0 = 0;
  s.sl = d;
  s.sh = static_cast<long long>(L) * d;
  s.sb = static_cast<long long>(H) * L * d;
  return s;
}

HeadStrides shape_strides(const svg_shape* sh) {
  const int L = sh->N * sh->F;
  if (sh->layout != SVG_LAYOUT_BLHD) return dense_strides(sh->B, sh->H, L, sh->d);
  HeadStrides s;
  s.H = sh->H;
  s.nb = sh->B;
  s.bh0 = 0;
  s.sl = static_cast<long long>(sh->H) * sh->d;
  s.sh = sh->d;
  s.sb = static_cast<long long>(L) * sh->H * sh->d;
  return s;
}

// The whole bf16 call folds the layout transformation into attention when
// that costs at most 3 % more attention work than the token-major copies.
// Not for [B, L, H, d] tensors: there one frame-group box, and one warp's
// output rows, span every frame of the tensor (frame stride F*H*d elements,
// 21.6 MB at HunyuanVideo, against F*d in [B, H, L, d]), and the fused
// attention ran 4 % slower than on [B, H, L, d] while the separate passes
// (token-major copies in [B, H, L, d]) ran as fast.
bool whole_call_fused(const svg_shape* s, int a2) {
  if (s->dtype != SVG_BF16 || a2 < 1 || s->layout == SVG_LAYOUT_BLHD) return false;
  return fused_layout_preferred(s->N, s->F, clamp_band(a2, s->N, s->N * s->F));
}

namespace {

svg_status status_word(int32_t* user, int** out, cudaStream_t stream) {
  if (user != nullptr) {
    *out = user;
    return SVG_OK;
  }
  return internal_status_word(out, stream);
}

}  // namespace

svg_status internal_status_word(int** out, cudaStream_t stream) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_internal_status);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetSymbolAddress(status)");
  e = cudaMemsetAsync(p, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_check(e, "cudaMemsetAsync(status)");
  *out = static_cast<int*>(p);
  return SVG_OK;
}

namespace {

// hs: layout of q, k, v, o; hsp: of the token-major (or, SVG2, cluster-
// permuted) copies.
svg_status run_attention(const svg_shape* s, const HeadStrides& hs, const HeadStrides& hsp, BandAttnArgs& a,
                         int32_t* status_dev, cudaStream_t stream, uint64_t wait_ns = kDefaultWaitNs) {
  a.hs = hs;
  a.hsp = hsp;
  a.B = s->B;
  a.H = s->H;
  a.L = s->N * s->F;
  a.d = s->d;
  a.dtype = s->dtype;
  a.scale = eff_scale(s);
  a.wait_ns = wait_ns;
  svg_status st = status_word(status_dev, &a.status, stream);
  if (st != SVG_OK) return st;
  if (s->dtype == SVG_BF16) return launch_attn_sm100(a, stream);
  if (s->dtype == SVG_TF32) return launch_attn_tf32(a, stream);
  return launch_attn_simt(a, stream);
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" {

int32_t svg_abi_version(void) { return SVG_ABI_VERSION; }

int32_t svg_debug_checks(void) { return SVG_DEBUG_BOUNDS ? 1 : 0; }

const char* svg_status_string(int32_t st) {
  switch (st) {
    case SVG_OK: return "SVG_OK";
    case SVG_ERR_INVALID_ARG: return "SVG_ERR_INVALID_ARG";
    case SVG_ERR_UNSUPPORTED: return "SVG_ERR_UNSUPPORTED";
    case SVG_ERR_CUDA: return "SVG_ERR_CUDA";
    case SVG_ERR_TIMEOUT: return "SVG_ERR_TIMEOUT";
    case SVG_ERR_WORKSPACE: return "SVG_ERR_WORKSPACE";
    default: return "SVG_ERR_UNKNOWN";
  }
}

const char* svg_last_error(void) { return g_last_error; }

svg_status svg_attn_tile(int32_t dtype, int32_t d, int32_t* Bq, int32_t* Bk) {
  if (Bq == nullptr || Bk == nullptr) return fail(SVG_ERR_INVALID_ARG, "NULL output");
  if (dtype == SVG_BF16) {
    if (d != 64 && d != 128) return fail(SVG_ERR_UNSUPPORTED, "bf16 supports d in {64, 128}");
    *Bq = kAttnBq;
    *Bk = kAttnBk;
    return SVG_OK;
  }
  if (dtype == SVG_FP32) {  // one row at a time, 32 keys per step
    *Bq = 1;
    *Bk = 32;
    return SVG_OK;
  }
  if (dtype == SVG_TF32) {  // 128-row query tiles, 128-key tiles
    if (d != 32 && d != 64 && d != 128) return fail(SVG_ERR_UNSUPPORTED, "tf32 supports d in {32, 64, 128}");
    *Bq = kAttnBq;
    *Bk = kAttnBk;
    return SVG_OK;
  }
  return fail(SVG_ERR_INVALID_ARG, "unknown dtype %d", dtype);
}

svg_status svg_block_list(int32_t L, int32_t G, int32_t a, int32_t Bq, int32_t Bk, int32_t* kb_lo, int32_t* kb_hi,
                          int32_t* full_lo, int32_t* full_hi) {
  if (L < 1 || G < 1 || a < 1 || Bq < 1 || Bk < 1) return fail(SVG_ERR_INVALID_ARG, "L, G, a, Bq, Bk must be >= 1");
  if (!kb_lo || !kb_hi || !full_lo || !full_hi) return fail(SVG_ERR_INVALID_ARG, "NULL output array");
  const int nq = (L + Bq - 1) / Bq;
  const long long aa = clamp_band(a, G, L);
  for (int qb = 0; qb < nq; ++qb) {
    const long long q0 = static_cast<long long>(qb) * Bq;
    const long long q1 = q0 + Bq < L ? q0 + Bq : L;
    const long long g_lo = q0 / G, g_hi = (q1 - 1) / G;
    // keys any row of the tile keeps: union of the rows' bands
    long long lo = (g_lo - aa + 1) * G;
    if (lo < 0) lo = 0;
    long long hi = (g_hi + aa) * G;
    if (hi > L) hi = L;
    kb_lo[qb] = static_cast<int32_t>(lo / Bk);
    kb_hi[qb] = static_cast<int32_t>((hi + Bk - 1) / Bk);
    // keys every row keeps: intersection of the rows' bands
    long long flo = (g_hi - aa + 1) * G;
    if (flo < 0) flo = 0;
    long long fhi = (g_lo + aa) * G;
    if (fhi > L) fhi = L;
    long long f0 = (flo + Bk - 1) / Bk;  // first tile starting at or after flo
    long long f1;                         // one past the last tile ending at or before fhi
    if (fhi >= L) f1 = (L + Bk - 1) / Bk;  // the ragged last tile ends at L
    else f1 = fhi / Bk;
    if (f1 < f0) f1 = f0;
    full_lo[qb] = static_cast<int32_t>(f0);
    full_hi[qb] = static_cast<int32_t>(f1);
  }
  return SVG_OK;
}

size_t svg_profile_workspace_size(const svg_shape* shape, int32_t S) {
  if (check_shape(shape) != SVG_OK) return 0;
  ProfileLayout lay;
  if (!profile_layout(shape->B, shape->H, shape->N * shape->F, shape->d, shape->dtype, S, &lay)) return 0;
  return lay.total;
}

size_t svg_workspace_size(const svg_shape* shape, int32_t n_temporal_heads_max) {
  if (check_shape(shape) != SVG_OK) return 0;
  if (n_temporal_heads_max < 0 || n_temporal_heads_max > shape->B * shape->H) return 0;
  const int L = shape->N * shape->F;
  const size_t prof = svg_profile_workspace_size(shape, L < 128 ? L : 128);
  if (prof == 0) return 0;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t elt = elem_size(shape->dtype);
  const size_t tensor = al(static_cast<size_t>(shape->B) * shape->H * L * shape->d * elt);
  return al(prof) + (n_temporal_heads_max > 0 ? 4 * tensor : 0);
}

svg_status svg_profile_heads(const svg_shape* shape, const void* q, const void* k, const void* v, int32_t a1,
                             int32_t a2, const int32_t* rows, int32_t S, float* mse, int8_t* label, void* workspace,
                             size_t workspace_bytes, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  return profile_heads_impl(shape, shape_strides(shape), q, k, v, a1, a2, rows, S, mse, label, workspace,
                            workspace_bytes, nullptr, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace svg {

svg_status profile_heads_impl(const svg_shape* shape, const HeadStrides& hs, const void* q, const void* k,
                              const void* v, int32_t a1, int32_t a2, const int32_t* rows, int32_t S, float* mse,
                              int8_t* label, void* workspace, size_t workspace_bytes, int32_t* status_out,
                              cudaStream_t stream, int chunk_len) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({q, k, v})) != SVG_OK) return st;
  if (!rows || !mse || !label || !workspace) return fail(SVG_ERR_INVALID_ARG, "NULL rows/mse/label/workspace");
  if (a1 < 1 || a2 < 1) return fail(SVG_ERR_INVALID_ARG, "a1 and a2 must be >= 1");
  const int L = shape->N * shape->F;
  if (S < 1 || S > 128 || S > L) return fail(SVG_ERR_INVALID_ARG, "S must be in [1, min(128, L)], got %d", S);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  ProfileLayout lay;
  profile_layout(shape->B, shape->H, L, shape->d, shape->dtype, S, &lay, 0, chunk_len);
  if (workspace_bytes < lay.total)
    return fail(SVG_ERR_WORKSPACE, "profile workspace %zu bytes < %zu required", workspace_bytes, lay.total);
  return launch_profile(shape->B, shape->H, shape->N, shape->F, shape->d, shape->dtype, eff_scale(shape), q, k, v, hs,
                        clamp_band(a1, 1, shape->N), clamp_band(a2, 1, shape->F), rows, S, mse, label, workspace, lay,
                        status_out, stream);
}

namespace {

// The layout transformation of up to three tensors, src laid out as ss and
// dst as ds; only heads whose label equals sel move (every head when label is
// NULL).
svg_status permute_impl(const svg_shape* s, int n, const void* const* src, void* const* dst, const HeadStrides& ss,
                        const HeadStrides& ds, const int8_t* label, bool to_token_major, cudaStream_t stream,
                        int sel = SVG_TEMPORAL) {
  return launch_permute(n, src, dst, s->B * s->H, s->N, s->F, s->d, static_cast<int>(elem_size(s->dtype)), ss, ds,
                        label, to_token_major, stream, sel);
}

// Block-sparse attention of labelled heads: spatial heads on (q, k, v) -> o
// laid out as hs, temporal heads on the token-major copies (qp, kp, vp) -> op
// laid out as hsp, or with fused != 0 temporal heads straight from (q, k, v)
// into o.
svg_status block_sparse_impl(const svg_shape* shape, const HeadStrides& hs, const HeadStrides& hsp, const void* q,
                             const void* k, const void* v, const void* qp, const void* kp, const void* vp, void* o,
                             void* op, const int8_t* label, int32_t a1, int32_t a2, int fused, int32_t* status_dev,
                             cudaStream_t stream) {
  const int L = shape->N * shape->F;
  BandAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  if (!fused) {
    a.qp = qp;
    a.kp = kp;
    a.vp = vp;
    a.op = op;
  }
  a.label = label;
  a.G0 = shape->F;
  a.a0 = clamp_band(a1, shape->F, L);
  a.G1 = shape->N;
  a.a1 = clamp_band(a2, shape->N, L);
  if (fused) {
    a.N = shape->N;
    a.fused = 1;
  }
  return run_attention(shape, hs, hsp, a, status_dev, stream);
}

// The whole call on `shape`'s heads, q, k, v, o laid out as hs (the
// token-major copies in the workspace are contiguous [B, H, L, d]).
svg_status sparse_3d_attn_impl(const svg_shape* shape, const HeadStrides& hs, const void* q, const void* k,
                               const void* v, void* o, int32_t a1, int32_t a2, const int32_t* rows, int32_t S,
                               float* mse, int8_t* label, void* workspace, size_t workspace_bytes,
                               int32_t* status_dev, cudaStream_t stream);

}  // namespace

}  // namespace svg

extern "C" {

svg_status svg_permute(const svg_shape* shape, const void* x, void* xp, const int8_t* label, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({x, xp})) != SVG_OK) return st;
  if (x == xp) return fail(SVG_ERR_INVALID_ARG, "permute cannot run in place");
  const void* src[1] = {x};
  void* dst[1] = {xp};
  const HeadStrides hs = shape_strides(shape);
  return permute_impl(shape, 1, src, dst, hs, hs, label, true, static_cast<cudaStream_t>(stream));
}

svg_status svg_permute_qkv(const svg_shape* shape, const void* q, const void* k, const void* v, void* qp, void* kp,
                           void* vp, const int8_t* label, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({q, k, v, qp, kp, vp})) != SVG_OK) return st;
  if (q == qp || k == kp || v == vp) return fail(SVG_ERR_INVALID_ARG, "permute cannot run in place");
  const void* src[3] = {q, k, v};
  void* dst[3] = {qp, kp, vp};
  const HeadStrides hs = shape_strides(shape);
  return permute_impl(shape, 3, src, dst, hs, hs, label, true, static_cast<cudaStream_t>(stream));
}

svg_status svg_unpermute(const svg_shape* shape, const void* xp, void* x, const int8_t* label, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({xp, x})) != SVG_OK) return st;
  if (x == xp) return fail(SVG_ERR_INVALID_ARG, "unpermute cannot run in place");
  const void* src[1] = {xp};
  void* dst[1] = {x};
  const HeadStrides hs = shape_strides(shape);
  return permute_impl(shape, 1, src, dst, hs, hs, label, false, static_cast<cudaStream_t>(stream));
}

svg_status svg_block_sparse_attn(const svg_shape* shape, const void* q, const void* k, const void* v, const void* qp,
                                 const void* kp, const void* vp, void* o, void* op, const int8_t* label, int32_t a1,
                                 int32_t a2, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({q, k, v, o, qp, kp, vp, op})) != SVG_OK) return st;
  if (label == nullptr) return fail(SVG_ERR_INVALID_ARG, "label is NULL");
  if (a1 < 1 || a2 < 1) return fail(SVG_ERR_INVALID_ARG, "a1 and a2 must be >= 1");
  const HeadStrides hs = shape_strides(shape);
  return block_sparse_impl(shape, hs, hs, q, k, v, qp, kp, vp, o, op, label, a1, a2, 0, status_dev,
                           static_cast<cudaStream_t>(stream));
}

svg_status svg_block_sparse_attn_fused(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                       const int8_t* label, int32_t a1, int32_t a2, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "the fused layout transformation runs in bf16 only");
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (label == nullptr) return fail(SVG_ERR_INVALID_ARG, "label is NULL");
  if (a1 < 1 || a2 < 1) return fail(SVG_ERR_INVALID_ARG, "a1 and a2 must be >= 1");
  const HeadStrides hs = shape_strides(shape);
  return block_sparse_impl(shape, hs, hs, q, k, v, nullptr, nullptr, nullptr, o, nullptr, label, a1, a2, 1, status_dev,
                           static_cast<cudaStream_t>(stream));
}

svg_status svg_banded_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o, int32_t G,
                           int32_t a_band, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (G < 1 || a_band < 1) return fail(SVG_ERR_INVALID_ARG, "G and a must be >= 1");
  const int L = shape->N * shape->F;
  if (G > L) G = L;
  BandAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.label = nullptr;
  a.G0 = G;
  a.a0 = clamp_band(a_band, G, L);
  a.G1 = a.G0;
  a.a1 = a.a0;
  const HeadStrides hs = shape_strides(shape);
  return run_attention(shape, hs, hs, a, status_dev, static_cast<cudaStream_t>(stream));
}

svg_status svg_dense_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                          int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  return svg_banded_attn(shape, q, k, v, o, shape->N * shape->F, 1, status_dev, stream);
}

size_t svg_sparse_3d_attn_workspace_size(const svg_shape* shape, int32_t a2, int32_t S) {
  if (check_shape(shape) != SVG_OK || a2 < 1) return 0;
  const size_t prof = svg_profile_workspace_size(shape, S);
  if (prof == 0) return 0;
  if (whole_call_fused(shape, a2)) return prof;  // layout transformation fused: no token-major copies
  const size_t t = static_cast<size_t>(shape->B) * shape->H * shape->N * shape->F * shape->d * elem_size(shape->dtype);
  const size_t t_al = (t + 255) / 256 * 256;
  return 4 * t_al + prof;
}

svg_status svg_sparse_3d_attn_plan(const svg_shape* shape, int32_t a2, int64_t* separate_tiles, int64_t* fused_tiles,
                                   int32_t* fused) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (a2 < 1) return fail(SVG_ERR_INVALID_ARG, "a2 must be >= 1");
  if (!separate_tiles || !fused_tiles || !fused) return fail(SVG_ERR_INVALID_ARG, "NULL output");
  long long sep = 0, fz = 0;
  token_major_tile_counts(shape->N, shape->F, clamp_band(a2, shape->N, shape->N * shape->F), &sep, &fz);
  *separate_tiles = sep;
  *fused_tiles = fz;
  *fused = whole_call_fused(shape, a2) ? 1 : 0;
  return SVG_OK;
}

svg_status svg_sparse_3d_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o, int32_t a1,
                              int32_t a2, const int32_t* rows, int32_t S, float* mse, int8_t* label, void* workspace,
                              size_t workspace_bytes, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  return sparse_3d_attn_impl(shape, shape_strides(shape), q, k, v, o, a1, a2, rows, S, mse, label, workspace,
                             workspace_bytes, status_dev, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace svg {
namespace {

svg_status sparse_3d_attn_impl(const svg_shape* shape, const HeadStrides& hs, const void* q, const void* k,
                               const void* v, void* o, int32_t a1, int32_t a2, const int32_t* rows, int32_t S,
                               float* mse, int8_t* label, void* workspace, size_t workspace_bytes,
                               int32_t* status_dev, cudaStream_t stream) {
  svg_status st;
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (!workspace) return fail(SVG_ERR_INVALID_ARG, "workspace is NULL");
  if (a1 < 1 || a2 < 1) return fail(SVG_ERR_INVALID_ARG, "a1 and a2 must be >= 1");
  const size_t need = svg_sparse_3d_attn_workspace_size(shape, a2, S);
  if (need == 0) return fail(SVG_ERR_INVALID_ARG, "S must be in [1, 128] and a2 >= 1");
  if (workspace_bytes < need) return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (whole_call_fused(shape, a2)) {
    if ((st = profile_heads_impl(shape, hs, q, k, v, a1, a2, rows, S, mse, label, workspace, workspace_bytes,
                                 status_dev, stream)) != SVG_OK)
      return st;
    return block_sparse_impl(shape, hs, hs, q, k, v, nullptr, nullptr, nullptr, o, nullptr, label, a1, a2, 1,
                             status_dev, stream);
  }
  const int L = shape->N * shape->F;
  const size_t t = static_cast<size_t>(shape->B) * shape->H * L * shape->d * elem_size(shape->dtype);
  const size_t t_al = (t + 255) / 256 * 256;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void *qp = w, *kp = w + t_al, *vp = w + 2 * t_al, *op = w + 3 * t_al;
  void* prof_ws = w + 4 * t_al;
  const size_t prof_bytes = workspace_bytes - 4 * t_al;
  const HeadStrides ws = dense_strides(shape->B, shape->H, L, shape->d);  // the token-major copies
  if ((st = profile_heads_impl(shape, hs, q, k, v, a1, a2, rows, S, mse, label, prof_ws, prof_bytes, status_dev,
                               stream)) != SVG_OK)
    return st;
  const void* src3[3] = {q, k, v};
  void* dst3[3] = {qp, kp, vp};
  if ((st = permute_impl(shape, 3, src3, dst3, hs, ws, label, true, stream)) != SVG_OK) return st;
  if ((st = block_sparse_impl(shape, hs, ws, q, k, v, qp, kp, vp, o, op, label, a1, a2, 0, status_dev, stream)) !=
      SVG_OK)
    return st;
  const void* src1[1] = {op};
  void* dst1[1] = {o};
  return permute_impl(shape, 1, src1, dst1, ws, hs, label, false, stream);
}

}  // namespace
}  // namespace svg

extern "C" {

svg_status svg_head_shard(int32_t n_heads, int32_t rank, int32_t world, int32_t* first, int32_t* count) {
  if (first == nullptr || count == nullptr) return fail(SVG_ERR_INVALID_ARG, "NULL output");
  if (n_heads < 0 || world < 1 || rank < 0 || rank >= world)
    return fail(SVG_ERR_INVALID_ARG, "need n_heads >= 0, world >= 1 and 0 <= rank < world (got %d, %d, %d)", n_heads,
                rank, world);
  const int32_t base = n_heads / world, extra = n_heads % world;
  *count = base + (rank < extra ? 1 : 0);
  *first = rank * base + (rank < extra ? rank : extra);
  return SVG_OK;
}

size_t svg_sparse_3d_attn_shard_workspace_size(const svg_shape* shape, int32_t rank, int32_t world, int32_t a2,
                                               int32_t S) {
  if (check_shape(shape) != SVG_OK) return 0;
  int32_t first = 0, count = 0;
  if (svg_head_shard(shape->B * shape->H, rank, world, &first, &count) != SVG_OK) return 0;
  if (count == 0) return 256;  // nothing to compute; a token workspace keeps the size query non-zero
  svg_shape local = *shape;
  local.B = 1;
  local.H = count;
  return svg_sparse_3d_attn_workspace_size(&local, a2, S);
}

svg_status svg_sparse_3d_attn_shard(const svg_shape* shape, int32_t rank, int32_t world, const void* q, const void* k,
                                    const void* v, void* o, int32_t a1, int32_t a2, const int32_t* rows, int32_t S,
                                    float* mse, int8_t* label, void* workspace, size_t workspace_bytes,
                                    int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  int32_t first = 0, count = 0;
  if ((st = svg_head_shard(shape->B * shape->H, rank, world, &first, &count)) != SVG_OK) return st;
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (!mse || !label) return fail(SVG_ERR_INVALID_ARG, "NULL mse/label");
  if (count == 0) return SVG_OK;  // more ranks than heads: this rank has none
  // heads are flattened over (b, h): this rank's heads are one contiguous
  // block of the [B, H] arrays (mse, label), and heads first .. first +
  // count - 1 of q, k, v, o in either layout, so the shard is the whole call
  // on that block
  svg_shape local = *shape;
  local.B = 1;
  local.H = count;
  HeadStrides hs = shape_strides(shape);
  hs.bh0 = first;
  return sparse_3d_attn_impl(&local, hs, q, k, v, o, a1, a2, rows, S, mse + 2 * static_cast<size_t>(first),
                             label + first, workspace, workspace_bytes, status_dev, static_cast<cudaStream_t>(stream));
}

svg_status svg_mixed_attn(const svg_shape* shape, const void* q, const void* k, const void* v, const void* qp,
                          const void* kp, const void* vp, void* o, void* op, const int8_t* mode, int32_t window,
                          int32_t md_half, int32_t stripe, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "mixed-pattern attention runs in bf16 only");
  if ((st = check_tensors({q, k, v, o, qp, kp, vp, op})) != SVG_OK) return st;
  if (mode == nullptr) return fail(SVG_ERR_INVALID_ARG, "mode is NULL");
  if (window < 0 || md_half < 0 || stripe < 1) return fail(SVG_ERR_INVALID_ARG, "window, md_half >= 0 and stripe >= 1");
  const int L = shape->N * shape->F;
  BandAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.qp = qp;
  a.kp = kp;
  a.vp = vp;
  a.op = op;
  a.modes = mode;
  a.G0 = L;
  a.a0 = 1;
  a.G1 = L;
  a.a1 = 1;
  a.win = window < L ? window : L;
  a.N = shape->N;
  a.md_a = clamp_band(md_half + 1, shape->N, L);
  a.stripe = stripe < L ? stripe : L;
  const HeadStrides hs = shape_strides(shape);
  return run_attention(shape, hs, hs, a, status_dev, static_cast<cudaStream_t>(stream));
}

svg_status svg_mixed_attn_fused(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                const int8_t* mode, int32_t window, int32_t md_half, int32_t stripe,
                                int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "mixed-pattern attention runs in bf16 only");
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (mode == nullptr) return fail(SVG_ERR_INVALID_ARG, "mode is NULL");
  if (window < 0 || md_half < 0 || stripe < 1) return fail(SVG_ERR_INVALID_ARG, "window, md_half >= 0 and stripe >= 1");
  const int L = shape->N * shape->F;
  BandAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.modes = mode;
  a.G0 = L;
  a.a0 = 1;
  a.G1 = L;
  a.a1 = 1;
  a.win = window < L ? window : L;
  a.N = shape->N;
  a.md_a = clamp_band(md_half + 1, shape->N, L);
  a.stripe = stripe < L ? stripe : L;
  a.fused = 1;
  const HeadStrides hs = shape_strides(shape);
  return run_attention(shape, hs, hs, a, status_dev, static_cast<cudaStream_t>(stream));
}

size_t svg_mixed_3d_attn_workspace_size(const svg_shape* shape) {
  if (check_shape(shape) != SVG_OK) return 0;
  const size_t t = static_cast<size_t>(shape->B) * shape->H * shape->N * shape->F * shape->d * elem_size(shape->dtype);
  return 4 * ((t + 255) / 256 * 256);
}

svg_status svg_mixed_3d_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                             const int8_t* mode, int32_t window, int32_t md_half, int32_t stripe, void* workspace,
                             size_t workspace_bytes, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (!workspace || !mode) return fail(SVG_ERR_INVALID_ARG, "workspace or mode is NULL");
  const size_t need = svg_mixed_3d_attn_workspace_size(shape);
  if (workspace_bytes < need) return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (window < 0 || md_half < 0 || stripe < 1) return fail(SVG_ERR_INVALID_ARG, "window, md_half >= 0 and stripe >= 1");
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "mixed-pattern attention runs in bf16 only");
  const size_t t_al = need / 4;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void *qp = w, *kp = w + t_al, *vp = w + 2 * t_al, *op = w + 3 * t_al;
  const int L = shape->N * shape->F;
  const HeadStrides hs = shape_strides(shape), ws = dense_strides(shape->B, shape->H, L, shape->d);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* src3[3] = {q, k, v};
  void* dst3[3] = {qp, kp, vp};
  if ((st = permute_impl(shape, 3, src3, dst3, hs, ws, mode, true, s, SVG_MODE_MULTIDIAG)) != SVG_OK) return st;
  BandAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.qp = qp;
  a.kp = kp;
  a.vp = vp;
  a.op = op;
  a.modes = mode;
  a.G0 = L;
  a.a0 = 1;
  a.G1 = L;
  a.a1 = 1;
  a.win = window < L ? window : L;
  a.N = shape->N;
  a.md_a = clamp_band(md_half + 1, shape->N, L);
  a.stripe = stripe < L ? stripe : L;
  if ((st = run_attention(shape, hs, ws, a, status_dev, s)) != SVG_OK) return st;
  const void* src1[1] = {op};
  void* dst1[1] = {o};
  return permute_impl(shape, 1, src1, dst1, ws, hs, mode, false, s, SVG_MODE_MULTIDIAG);
}

size_t svg_semantic_attn_workspace_size(const svg_shape* shape, int32_t Cq, int32_t Ck) {
  if (check_shape(shape) != SVG_OK || shape->dtype != SVG_BF16) return 0;
  if (Cq < 1 || Ck < 1 || Cq > 1024 || Ck > 1024) return 0;
  return svg2_sizes(shape->B * shape->H, shape->N * shape->F, Cq, Ck, shape->d).total;
}

svg_status svg_semantic_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                             const int32_t* assign_q, const int32_t* assign_k, int32_t Cq, int32_t Ck, float p,
                             uint32_t* selected, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                             void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "semantic-aware attention runs in bf16 only");
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (!assign_q || !assign_k || !selected || !workspace) return fail(SVG_ERR_INVALID_ARG, "NULL argument");
  if (Cq < 1 || Ck < 1 || Cq > 1024 || Ck > 1024)
    return fail(SVG_ERR_INVALID_ARG, "cluster counts must be in [1, 1024], got %d, %d", Cq, Ck);
  if (!(p > 0.f && p <= 1.f)) return fail(SVG_ERR_INVALID_ARG, "p must be in (0, 1]");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const int BH = shape->B * shape->H, L = shape->N * shape->F, d = shape->d;
  const Svg2Sizes z = svg2_sizes(BH, L, Cq, Ck, d);
  if (workspace_bytes < z.total) return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, z.total);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int32_t* hist = reinterpret_cast<int32_t*>(w);
  w += z.hist;
  int32_t* perm_q = reinterpret_cast<int32_t*>(w);
  int32_t* cid_q = reinterpret_cast<int32_t*>(w + z.perm);
  int32_t* perm_k = reinterpret_cast<int32_t*>(w + 2 * z.perm);
  int32_t* cid_k = reinterpret_cast<int32_t*>(w + 3 * z.perm);
  w += 4 * z.perm;
  int32_t* off_q = reinterpret_cast<int32_t*>(w);
  w += z.off_q;
  int32_t* off_k = reinterpret_cast<int32_t*>(w);
  w += z.off_k;
  float* mu_q = reinterpret_cast<float*>(w);
  w += z.mu_q;
  float* mu_k = reinterpret_cast<float*>(w);
  w += z.mu_k;
  void* qp = w;
  void* kp = w + z.tensor;
  void* vp = w + 2 * z.tensor;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* dev_status = nullptr;
  if ((st = status_word(status_dev, &dev_status, s)) != SVG_OK) return st;
  if ((st = svg2_sort(assign_q, BH, L, Cq, z.nblk, hist, perm_q, cid_q, off_q, dev_status, s)) != SVG_OK) return st;
  if ((st = svg2_sort(assign_k, BH, L, Ck, z.nblk, hist, perm_k, cid_k, off_k, dev_status, s)) != SVG_OK) return st;
  const HeadStrides hs = shape_strides(shape), ws = dense_strides(shape->B, shape->H, L, d);
  if ((st = svg2_gather(q, hs, perm_q, qp, BH, L, d, s)) != SVG_OK) return st;
  if ((st = svg2_gather(k, hs, perm_k, kp, BH, L, d, s)) != SVG_OK) return st;
  if ((st = svg2_gather(v, hs, perm_k, vp, BH, L, d, s)) != SVG_OK) return st;
  if ((st = svg2_centroids(qp, off_q, BH, L, Cq, d, mu_q, s)) != SVG_OK) return st;
  if ((st = svg2_centroids(kp, off_k, BH, L, Ck, d, mu_k, s)) != SVG_OK) return st;
  if ((st = svg2_topp(mu_q, mu_k, off_k, BH, Cq, Ck, d, eff_scale(shape), p, selected, s)) != SVG_OK) return st;
  BandAttnArgs a{};
  a.q = qp;
  a.k = kp;
  a.v = vp;
  a.o = o;
  a.G0 = L;
  a.a0 = 1;
  a.G1 = L;
  a.a1 = 1;
  a.s2 = 1;
  a.s2_Cq = Cq;
  a.s2_Ck = Ck;
  a.s2_cid = cid_q;
  a.s2_perm = perm_q;
  a.s2_koff = off_k;
  a.s2_sel = selected;
  return run_attention(shape, hs, ws, a, dev_status, s);
}

size_t svg_kmeans_workspace_size(const svg_shape* shape, int32_t C) {
  if (check_shape(shape) != SVG_OK || shape->dtype != SVG_BF16 || C < 1 || C > 512) return 0;
  return kmeans_workspace_bytes(shape->B * shape->H, shape->N * shape->F, C, shape->d);
}

svg_status svg_kmeans(const svg_shape* shape, const void* x, int32_t C, int32_t iters, int32_t* assign,
                      float* centroids, void* workspace, size_t workspace_bytes, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "k-means runs on bf16 rows only");
  if ((st = check_tensors({x})) != SVG_OK) return st;
  if (!assign || !centroids || !workspace) return fail(SVG_ERR_INVALID_ARG, "NULL assign/centroids/workspace");
  if (C < 1 || C > 512) return fail(SVG_ERR_INVALID_ARG, "C must be in [1, 512], got %d", C);
  if (iters < 1) return fail(SVG_ERR_INVALID_ARG, "iters must be >= 1");
  const int L = shape->N * shape->F;
  if (C > L) return fail(SVG_ERR_INVALID_ARG, "C = %d exceeds the %d rows", C, L);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t need = svg_kmeans_workspace_size(shape, C);
  if (workspace_bytes < need) return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, need);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* dev_status = nullptr;
  if ((st = status_word(status_dev, &dev_status, s)) != SVG_OK) return st;
  return launch_kmeans(x, shape_strides(shape), shape->B * shape->H, L, C, shape->d, iters, assign, centroids, workspace,
                       dev_status, s);
}

size_t svg_semantic_3d_attn_workspace_size(const svg_shape* shape, int32_t Cq, int32_t Ck) {
  const size_t km_q = svg_kmeans_workspace_size(shape, Cq), km_k = svg_kmeans_workspace_size(shape, Ck);
  const size_t at = svg_semantic_attn_workspace_size(shape, Cq, Ck);
  if (km_q == 0 || km_k == 0 || at == 0) return 0;
  const size_t BH = static_cast<size_t>(shape->B) * shape->H;
  const size_t cent = ((BH * (Cq > Ck ? Cq : Ck) * shape->d * 4) + 255) / 256 * 256;
  const size_t km = km_q > km_k ? km_q : km_k;
  return (km > at ? km : at) + cent;
}

svg_status svg_semantic_3d_attn(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                int32_t Cq, int32_t Ck, int32_t iters, float p, int32_t* assign_q, int32_t* assign_k,
                                uint32_t* selected, void* workspace, size_t workspace_bytes, int32_t* status_dev,
                                void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  const size_t need = svg_semantic_3d_attn_workspace_size(shape, Cq, Ck);
  if (need == 0) return fail(SVG_ERR_INVALID_ARG, "bad shape (bf16 only) or cluster counts (1..512)");
  if (!workspace) return fail(SVG_ERR_INVALID_ARG, "workspace is NULL");
  if (workspace_bytes < need) return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, need);
  const size_t BH = static_cast<size_t>(shape->B) * shape->H;
  const size_t cent = ((BH * (Cq > Ck ? Cq : Ck) * shape->d * 4) + 255) / 256 * 256;
  float* centroids = static_cast<float*>(workspace);  // scratch: the k-means centroids (unused afterwards)
  void* rest = static_cast<uint8_t*>(workspace) + cent;
  const size_t rest_bytes = workspace_bytes - cent;
  if ((st = svg_kmeans(shape, q, Cq, iters, assign_q, centroids, rest, rest_bytes, status_dev, stream)) != SVG_OK)
    return st;
  if ((st = svg_kmeans(shape, k, Ck, iters, assign_k, centroids, rest, rest_bytes, status_dev, stream)) != SVG_OK)
    return st;
  return svg_semantic_attn(shape, q, k, v, o, assign_q, assign_k, Cq, Ck, p, selected, rest, rest_bytes, status_dev,
                           stream);
}

size_t svg_mode_search_workspace_size(const svg_shape* shape, int32_t S) {
  if (check_shape(shape) != SVG_OK || shape->dtype != SVG_BF16) return 0;
  ProfileLayout lay;
  if (!profile_layout(shape->B, shape->H, shape->N * shape->F, shape->d, shape->dtype, S, &lay)) return 0;
  return lay.total + lay.part_bytes;
}

svg_status svg_mode_search(const svg_shape* shape, const void* q, const void* k, const void* v, const int32_t* rows,
                           int32_t S, int32_t window, int32_t md_half, int32_t stripe, float lambda, float epsilon,
                           float* loss, int8_t* mode, void* workspace, size_t workspace_bytes, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "the mode search runs in bf16 only");
  if ((st = check_tensors({q, k, v})) != SVG_OK) return st;
  if (!rows || !loss || !mode || !workspace) return fail(SVG_ERR_INVALID_ARG, "NULL rows/loss/mode/workspace");
  if (window < 0 || md_half < 0 || stripe < 1) return fail(SVG_ERR_INVALID_ARG, "window, md_half >= 0 and stripe >= 1");
  if (!(lambda >= 0.f) || !(epsilon >= 0.f)) return fail(SVG_ERR_INVALID_ARG, "lambda and epsilon must be >= 0");
  const int L = shape->N * shape->F;
  if (S < 1 || S > 128 || S > L) return fail(SVG_ERR_INVALID_ARG, "S must be in [1, min(128, L)], got %d", S);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  ProfileLayout lay;
  profile_layout(shape->B, shape->H, L, shape->d, shape->dtype, S, &lay);
  if (workspace_bytes < lay.total + lay.part_bytes)
    return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, lay.total + lay.part_bytes);
  double* part2 = reinterpret_cast<double*>(static_cast<uint8_t*>(workspace) + lay.total);
  return launch_mode_search(shape->B, shape->H, shape->N, shape->F, shape->d, eff_scale(shape), q, k, v,
                            shape_strides(shape), rows, S,
                            window < L ? window : L, md_half < shape->F ? md_half : shape->F, stripe < L ? stripe : L,
                            lambda, epsilon, loss, mode, workspace, lay, part2, static_cast<cudaStream_t>(stream));
}

svg_status svg_selftest_wait_bound(const svg_shape* shape, const void* q, const void* k, const void* v, void* o,
                                   uint64_t wait_ns, int32_t* status_dev, void* stream) {
  svg_status st = check_shape(shape);
  if (st != SVG_OK) return st;
  if (shape->dtype != SVG_BF16) return fail(SVG_ERR_UNSUPPORTED, "the self-test runs the bf16 tensor-core kernel");
  if ((st = check_tensors({q, k, v, o})) != SVG_OK) return st;
  if (status_dev == nullptr) return fail(SVG_ERR_INVALID_ARG, "status_dev is required");
  if (wait_ns < 1000000ull || wait_ns > 10000000000ull)
    return fail(SVG_ERR_INVALID_ARG, "wait_ns must be in [1 ms, 10 s]");
  const int L = shape->N * shape->F;
  BandAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.label = nullptr;
  a.G0 = L;
  a.a0 = 1;
  a.G1 = L;
  a.a1 = 1;
  a.withhold_loads = 1;
  const HeadStrides hs = shape_strides(shape);
  return run_attention(shape, hs, hs, a, status_dev, static_cast<cudaStream_t>(stream), wait_ns);
}

}  // extern "C"
