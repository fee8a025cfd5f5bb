// attn_simt.cu -- banded attention for fp32 inputs on the CUDA cores.
//
// fp32 tensors (small shapes) do not go through the bf16 tensor-core kernel;
// this kernel computes the same banded attention in fp32 FMA arithmetic:
// keep (x, y) iff |floor(x/G) - floor(y/G)| < a ("Sparse Video-Gen", Spatial
// Head with G = F, a = a1; Temporal Head after the token-major layout
// transformation with G = N, a = a2).  One warp owns one query row and walks
// the row's contiguous key interval 32 keys at a time with an online softmax.
#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kSimtWarps = 8;

template <int D>
__global__ void __launch_bounds__(kSimtWarps * 32)
    attn_simt_kernel(const float* __restrict__ q0, const float* __restrict__ k0, const float* __restrict__ v0,
                     float* __restrict__ o0, const float* __restrict__ q1, const float* __restrict__ k1,
                     const float* __restrict__ v1, float* __restrict__ o1, const HeadStrides s0, const HeadStrides s1,
                     const int8_t* __restrict__ label, int BH, int L, int G0, int a0, int G1, int a1, float sl2) {
  constexpr int PER = D / 32;
  __shared__ float sq[kSimtWarps][D];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long gid = static_cast<long long>(blockIdx.x) * kSimtWarps + warp;
  if (gid >= static_cast<long long>(BH) * L) return;
  const int bh = static_cast<int>(gid / L);
  const int x = static_cast<int>(gid - static_cast<long long>(bh) * L);
  const int lab = (label != nullptr && label[bh] == SVG_TEMPORAL) ? 1 : 0;  // any other label runs spatial
  const int G = lab ? G1 : G0, a = lab ? a1 : a0;
  const HeadStrides& hs = lab ? s1 : s0;  // (q0, k0, v0, o0) and (q1, k1, v1, o1) layouts
  const long long hoff = hs.head(bh), sl = hs.sl;
  const float* q = (lab ? q1 : q0) + hoff;
  const float* k = (lab ? k1 : k0) + hoff;
  const float* v = (lab ? v1 : v0) + hoff;
  float* o = (lab ? o1 : o0) + hoff;

  const long long g = x / G;
  const int lo = static_cast<int>(max(0LL, (g - a + 1) * G));
  const int hi = static_cast<int>(min(static_cast<long long>(L), (g + a) * G));

  for (int c = lane; c < D; c += 32) sq[warp][c] = q[x * sl + c] * sl2;
  __syncwarp();

  float m = -INFINITY, l = 0.f, acc[PER];
#pragma unroll
  for (int t = 0; t < PER; ++t) acc[t] = 0.f;

  for (int y0 = lo; y0 < hi; y0 += 32) {
    const int y = y0 + lane;
    float s = -INFINITY;
    if (y < hi) {
      const float* kr = k + y * sl;
      float dot = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) dot = fmaf(sq[warp][c], kr[c], dot);
      s = dot;  // already in log2 units
    }
    float mx = s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float m_new = fmaxf(m, mx);
    const float alpha = ex2_approx(m - m_new);  // m = -inf on the first block -> 0
    const float p = ex2_approx(s - m_new);      // masked / out of range -> 0
    float ps = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * alpha + ps;
#pragma unroll
    for (int t = 0; t < PER; ++t) acc[t] *= alpha;
    const int nvalid = min(32, hi - y0);
    for (int jj = 0; jj < nvalid; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const float* vr = v + (y0 + jj) * sl;
#pragma unroll
      for (int t = 0; t < PER; ++t) acc[t] = fmaf(pj, vr[lane + 32 * t], acc[t]);
    }
    m = m_new;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int t = 0; t < PER; ++t) o[x * sl + lane + 32 * t] = acc[t] * inv;
}

template <int D>
svg_status launch_simt_d(const BandAttnArgs& a, cudaStream_t stream) {
  const long long rows = static_cast<long long>(a.B) * a.H * a.L;
  const long long blocks = (rows + kSimtWarps - 1) / kSimtWarps;
  if (blocks > 0x7fffffffLL) return fail(SVG_ERR_UNSUPPORTED, "too many rows for the fp32 kernel");
  const float sl2 = a.scale * 1.4426950408889634f;
  attn_simt_kernel<D><<<static_cast<unsigned>(blocks), kSimtWarps * 32, 0, stream>>>(
      static_cast<const float*>(a.q), static_cast<const float*>(a.k), static_cast<const float*>(a.v),
      static_cast<float*>(a.o), static_cast<const float*>(a.qp), static_cast<const float*>(a.kp),
      static_cast<const float*>(a.vp), static_cast<float*>(a.op), a.hs, a.label ? a.hsp : a.hs, a.label, a.B * a.H,
      a.L, a.G0, a.a0, a.G1, a.a1, sl2);
  return cuda_check(cudaGetLastError(), "fp32 attention launch");
}

}  // namespace

svg_status launch_attn_simt(const BandAttnArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 32: return launch_simt_d<32>(a, stream);
    case 64: return launch_simt_d<64>(a, stream);
    case 128: return launch_simt_d<128>(a, stream);
    default: return fail(SVG_ERR_UNSUPPORTED, "fp32 attention supports d in {32, 64, 128}, got %d", a.d);
  }
}

}  // namespace svg
