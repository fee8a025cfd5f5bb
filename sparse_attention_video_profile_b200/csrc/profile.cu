// profile.cu -- online profiling ("Sparse Video-Gen", Weakness 1 answer on
// online profiling: run right before each 3D attention call; "Sparse VideoGen
// ...", Abstract: classify heads spatial or temporal online).
//
// For the S sampled query rows of every head, the exact attention output is
// computed three times over all L keys -- unmasked (O_d), under the spatial
// mask |i_x - i_y| < a1 (O_s) and under the temporal mask |j_x - j_y| < a2
// (O_t) -- and the head is labelled by the lower of
//   mse_s = mean (O_s - O_d)^2,  mse_t = mean (O_t - O_d)^2.
//
// Stage 1 (profile_mma_kernel, bf16): the key axis is split into chunks so
// that B*H*chunks*row-blocks CTAs cover the GPU; each CTA streams its chunk
// of K and V once through shared memory (cp.async double buffer, XOR
// swizzle) and keeps, per sampled row, three online-softmax states (max,
// sum, unnormalised output) updated from one shared Q K^T tile.  The
// products use mma.sync m16n8k16 bf16 -> fp32.  Partial (max, sum, output)
// triples go to the workspace.
// Stage 2 (profile_combine_kernel): per head, merges the chunk partials in a
// fixed order, forms O_d, O_s, O_t, and reduces the squared differences in
// fp64 with a fixed tree -- so repeated calls return identical bits.
// fp32 inputs use profile_simt_kernel (one warp per row, all keys) for stage
// 1 and the same stage 2.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kKT = 64;  // keys per tile in stage 1

struct ProfParams {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* rows;
  float* ws_o;   // [BH][nch][3][S_pad][D]
  float* ws_ml;  // [BH][nch][3][S_pad][2]  (max in log2 units, sum)
  int BH, L, N, F, S, S_pad, nch, chunk;
  int a1, a2;
  float sl2;
};

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Byte offset of 16-byte chunk c of row `row` in a [rows][D] bf16 tile whose
// chunks are XOR-swizzled by the row's low three bits (conflict-free
// ldmatrix on both the row and the transposed access).
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int c) {
  return static_cast<uint32_t>(row * D * 2 + ((c ^ (row & 7)) << 4));
}

template <int D>
struct ProfCfg {
  static constexpr int DS = D / 64;      // warps sharing a row block, one per 64 output columns
  static constexpr int RG = 4 / DS;      // 16-row blocks per CTA
  static constexpr int ROWS = 16 * RG;   // sampled rows per CTA
  static constexpr int TILE = kKT * D * 2;
  static constexpr int SMEM = ROWS * D * 2 + 4 * TILE + 4 * kKT * 4;
};

template <int D>
__global__ void __launch_bounds__(128) profile_mma_kernel(const ProfParams p) {
  using C = ProfCfg<D>;
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::ROWS * D * 2;  // [2][TILE]
  uint8_t* sV = sK + 2 * C::TILE;        // [2][TILE]
  int* sIY = reinterpret_cast<int*>(sV + 2 * C::TILE);  // [2][kKT]
  int* sJY = sIY + 2 * kKT;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rg = warp / C::DS, ds = warp % C::DS;
  const int row_base = blockIdx.x * C::ROWS;  // first sampled-row index of this CTA
  const int chunk = blockIdx.y;
  const int bh = blockIdx.z;
  const size_t hoff = static_cast<size_t>(bh) * p.L * D;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(p.q) + hoff;
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(p.k) + hoff;
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(p.v) + hoff;
  const int y_begin = chunk * p.chunk;
  const int y_end = min(p.L, y_begin + p.chunk);
  const int ntiles = (y_end - y_begin + kKT - 1) / kKT;

  // gather the CTA's sampled query rows (padding rows repeat the last row)
  for (int e = tid; e < C::ROWS * CPR; e += 128) {
    const int r = e / CPR, c = e % CPR;
    const int s = min(row_base + r, p.S - 1);
    const int x = min(max(p.rows[s], 0), p.L - 1);
    cp_async16(smem_u32(sQ) + swz<D>(r, c), q + static_cast<size_t>(x) * D + c * 8, true);
  }
  auto load_tile = [&](int t, int stage) {
    const int y0 = y_begin + t * kKT;
    const uint32_t kb = smem_u32(sK + stage * C::TILE), vb = smem_u32(sV + stage * C::TILE);
    for (int e = tid; e < kKT * CPR; e += 128) {
      const int r = e / CPR, c = e % CPR;
      const int y = y0 + r;
      const bool ok = y < p.L;
      const size_t off = static_cast<size_t>(ok ? y : 0) * D + c * 8;
      cp_async16(kb + swz<D>(r, c), k + off, ok);
      cp_async16(vb + swz<D>(r, c), v + off, ok);
    }
    if (tid < kKT) {
      const int y = y0 + tid;
      sIY[stage * kKT + tid] = y / p.F;
      sJY[stage * kKT + tid] = y % p.F;
    }
  };
  load_tile(0, 0);
  cp_async_commit();

  // the two rows this thread owns in the mma fragments
  const int g = lane >> 2, tq = lane & 3;
  int ir[2], jr[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int s = min(row_base + rg * 16 + g + 8 * h, p.S - 1);
    const int x = min(max(p.rows[s], 0), p.L - 1);
    ir[h] = x / p.F;
    jr[h] = x % p.F;
  }

  float m[3][2], l[3][2], o[3][8][4];
#pragma unroll
  for (int vv = 0; vv < 3; ++vv)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      m[vv][h] = -INFINITY;
      l[vv][h] = 0.f;
    }
#pragma unroll
  for (int vv = 0; vv < 3; ++vv)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[vv][nt][e] = 0.f;

  uint32_t qf[D / 16][4];
  const float sl2 = p.sl2;

  for (int t = 0; t < ntiles; ++t) {
    const int stage = t & 1;
    if (t + 1 < ntiles) {
      load_tile(t + 1, stage ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(qf[kk], smem_u32(sQ) + swz<D>(rg * 16 + (lane & 15), kk * 2 + (lane >> 4)));
    }
    const uint32_t kb = smem_u32(sK + stage * C::TILE), vb = smem_u32(sV + stage * C::TILE);
    // S = Q K^T for this warp's 16 rows x 64 keys
    float sacc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b[4];
        ldsm_x4(b, kb + swz<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)));
        mma_bf16(sacc[2 * np], qf[kk], b[0], b[1]);
        mma_bf16(sacc[2 * np + 1], qf[kk], b[2], b[3]);
      }
    }
    // frame / position of this thread's 16 key columns
    const int y0 = y_begin + t * kKT;
    int iy[16], jy[16];
    bool in_chunk[16];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = nt * 8 + tq * 2 + e;
        iy[nt * 2 + e] = sIY[stage * kKT + c];
        jy[nt * 2 + e] = sJY[stage * kKT + c];
        in_chunk[nt * 2 + e] = (y0 + c) < y_end;
      }
#pragma unroll
    for (int vv = 0; vv < 3; ++vv) {
      uint32_t pf[4][4];  // P as A fragments, 4 k-steps of 16 keys
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float sv[16];
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int cc = nt * 2 + e;
            bool ok = in_chunk[cc];
            if (vv == 1) ok = ok && (abs(ir[h] - iy[cc]) < p.a1);
            if (vv == 2) ok = ok && (abs(jr[h] - jy[cc]) < p.a2);
            sv[cc] = ok ? sacc[nt][2 * h + e] : -INFINITY;
            mx = fmaxf(mx, sv[cc]);
          }
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_old = m[vv][h];
        const float m_new = fmaxf(m_old, mx);
        const float alpha = (m_new == m_old) ? 1.f : ex2_approx((m_old - m_new) * sl2);
        const float nb = (m_new == -INFINITY) ? 0.f : -m_new * sl2;
        float pv[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) pv[cc] = ex2_approx(fmaf(sv[cc], sl2, nb));  // -inf -> 0
        m[vv][h] = m_new;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          o[vv][nt][2 * h] *= alpha;
          o[vv][nt][2 * h + 1] *= alpha;
        }
        float ps = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          pf[ks][h] = pack_bf16x2(pv[4 * ks + 0], pv[4 * ks + 1]);      // keys 16ks + 2tq (+1)
          pf[ks][2 + h] = pack_bf16x2(pv[4 * ks + 2], pv[4 * ks + 3]);  // keys 16ks + 8 + 2tq (+1)
          // sum the bf16-rounded weights the P V product uses
          ps += bf16lo_f32(pf[ks][h]) + bf16hi_f32(pf[ks][h]) + bf16lo_f32(pf[ks][2 + h]) +
                bf16hi_f32(pf[ks][2 + h]);
        }
        l[vv][h] = l[vv][h] * alpha + ps;
      }
      // O_v += P_v V over this warp's 64 output columns
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b[4];
          ldsm_x4_t(b, vb + swz<D>(ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), ds * 8 + np * 2 + (lane >> 4)));
          mma_bf16(o[vv][2 * np], pf[ks], b[0], b[1]);
          mma_bf16(o[vv][2 * np + 1], pf[ks], b[2], b[3]);
        }
      }
    }
    __syncthreads();
  }

  // write partials
#pragma unroll
  for (int vv = 0; vv < 3; ++vv) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float ls = l[vv][h];
      ls += __shfl_xor_sync(0xffffffffu, ls, 1);
      ls += __shfl_xor_sync(0xffffffffu, ls, 2);
      const int s = row_base + rg * 16 + g + 8 * h;
      const size_t base = ((static_cast<size_t>(bh) * p.nch + chunk) * 3 + vv) * p.S_pad + s;
      float* orow = p.ws_o + base * D + ds * 64;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        *reinterpret_cast<float2*>(orow + nt * 8 + tq * 2) = make_float2(o[vv][nt][2 * h], o[vv][nt][2 * h + 1]);
      if (tq == 0 && ds == 0) {
        const float mm = m[vv][h];
        p.ws_ml[base * 2 + 0] = (mm == -INFINITY) ? -INFINITY : mm * sl2;
        p.ws_ml[base * 2 + 1] = ls;
      }
    }
  }
}

// fp32 stage 1: one warp per (head, sampled row), all keys, chunk count 1.
template <int D>
__global__ void __launch_bounds__(128) profile_simt_kernel(const ProfParams p) {
  constexpr int PER = D / 32;
  __shared__ float sq[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x * 4 + warp;
  const int bh = blockIdx.y;
  if (s >= p.S_pad) return;
  const size_t hoff = static_cast<size_t>(bh) * p.L * D;
  const float* q = static_cast<const float*>(p.q) + hoff;
  const float* k = static_cast<const float*>(p.k) + hoff;
  const float* v = static_cast<const float*>(p.v) + hoff;
  const int x = min(max(p.rows[min(s, p.S - 1)], 0), p.L - 1);
  const int ir = x / p.F, jr = x % p.F;
  for (int c = lane; c < D; c += 32) sq[warp][c] = q[static_cast<size_t>(x) * D + c] * p.sl2;
  __syncwarp();
  float m[3], l[3], acc[3][PER];
#pragma unroll
  for (int vv = 0; vv < 3; ++vv) {
    m[vv] = -INFINITY;
    l[vv] = 0.f;
#pragma unroll
    for (int t = 0; t < PER; ++t) acc[vv][t] = 0.f;
  }
  for (int y0 = 0; y0 < p.L; y0 += 32) {
    const int y = y0 + lane;
    float sc = -INFINITY;
    int iy = -1, jy = -1;
    if (y < p.L) {
      const float* kr = k + static_cast<size_t>(y) * D;
      float dot = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) dot = fmaf(sq[warp][c], kr[c], dot);
      sc = dot;
      iy = y / p.F;
      jy = y % p.F;
    }
    float pv[3];
#pragma unroll
    for (int vv = 0; vv < 3; ++vv) {
      bool ok = y < p.L;
      if (vv == 1) ok = ok && abs(ir - iy) < p.a1;
      if (vv == 2) ok = ok && abs(jr - jy) < p.a2;
      const float sv = ok ? sc : -INFINITY;
      float mx = sv;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[vv], mx);
      const float alpha = (m_new == m[vv]) ? 1.f : ex2_approx(m[vv] - m_new);
      const float pp = (m_new == -INFINITY) ? 0.f : ex2_approx(sv - m_new);
      float ps = pp;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[vv] = l[vv] * alpha + ps;
      m[vv] = m_new;
#pragma unroll
      for (int t = 0; t < PER; ++t) acc[vv][t] *= alpha;
      pv[vv] = pp;
    }
    const int nvalid = min(32, p.L - y0);
    for (int jj = 0; jj < nvalid; ++jj) {
      const float* vr = v + static_cast<size_t>(y0 + jj) * D;
      float vals[PER];
#pragma unroll
      for (int t = 0; t < PER; ++t) vals[t] = vr[lane + 32 * t];
#pragma unroll
      for (int vv = 0; vv < 3; ++vv) {
        const float pj = __shfl_sync(0xffffffffu, pv[vv], jj);
#pragma unroll
        for (int t = 0; t < PER; ++t) acc[vv][t] = fmaf(pj, vals[t], acc[vv][t]);
      }
    }
  }
#pragma unroll
  for (int vv = 0; vv < 3; ++vv) {
    const size_t base = (static_cast<size_t>(bh) * 3 + vv) * p.S_pad + s;  // nch == 1
#pragma unroll
    for (int t = 0; t < PER; ++t) p.ws_o[base * D + lane + 32 * t] = acc[vv][t];
    if (lane == 0) {
      p.ws_ml[base * 2 + 0] = m[vv];  // already in log2 units
      p.ws_ml[base * 2 + 1] = l[vv];
    }
  }
}

constexpr int kCombineThreads = 256;

// Stage 2: merge chunk partials, form O_d / O_s / O_t, reduce the MSEs.
__global__ void __launch_bounds__(kCombineThreads)
    profile_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml, int S, int S_pad, int D,
                           int nch, float* __restrict__ mse, int8_t* __restrict__ label) {
  __shared__ double red[2][kCombineThreads];
  const int bh = blockIdx.x;
  double acc_s = 0.0, acc_t = 0.0;
  const int total = S * D;
  for (int e = threadIdx.x; e < total; e += kCombineThreads) {
    const int s = e / D, c = e % D;
    float ov[3];
#pragma unroll
    for (int vv = 0; vv < 3; ++vv) {
      float M = -INFINITY;
      for (int ch = 0; ch < nch; ++ch) {
        const size_t base = ((static_cast<size_t>(bh) * nch + ch) * 3 + vv) * S_pad + s;
        M = fmaxf(M, ws_ml[base * 2]);
      }
      float Ls = 0.f, Os = 0.f;
      if (M != -INFINITY) {
        for (int ch = 0; ch < nch; ++ch) {
          const size_t base = ((static_cast<size_t>(bh) * nch + ch) * 3 + vv) * S_pad + s;
          const float mc = ws_ml[base * 2];
          if (mc == -INFINITY) continue;
          const float w = ex2_approx(mc - M);
          Ls = fmaf(ws_ml[base * 2 + 1], w, Ls);
          Os = fmaf(ws_o[base * D + c], w, Os);
        }
      }
      ov[vv] = Ls > 0.f ? Os / Ls : 0.f;
    }
    const double dsp = static_cast<double>(ov[1]) - ov[0];
    const double dtp = static_cast<double>(ov[2]) - ov[0];
    acc_s += dsp * dsp;
    acc_t += dtp * dtp;
  }
  red[0][threadIdx.x] = acc_s;
  red[1][threadIdx.x] = acc_t;
  __syncthreads();
  for (int w = kCombineThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      red[0][threadIdx.x] += red[0][threadIdx.x + w];
      red[1][threadIdx.x] += red[1][threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double n = static_cast<double>(total);
    const float ms = static_cast<float>(red[0][0] / n), mt = static_cast<float>(red[1][0] / n);
    mse[bh * 2 + 0] = ms;
    mse[bh * 2 + 1] = mt;
    label[bh] = (mt < ms) ? SVG_TEMPORAL : SVG_SPATIAL;
  }
}

template <int D>
svg_status launch_stage1_bf16(const ProfParams& p, cudaStream_t stream) {
  using C = ProfCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(profile_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute(profile smem)");
  dim3 grid(p.S_pad / C::ROWS, p.nch, p.BH);
  profile_mma_kernel<D><<<grid, 128, C::SMEM, stream>>>(p);
  return cuda_check(cudaGetLastError(), "profile launch");
}

template <int D>
svg_status launch_stage1_f32(const ProfParams& p, cudaStream_t stream) {
  dim3 grid((p.S_pad + 3) / 4, p.BH);
  profile_simt_kernel<D><<<grid, 128, 0, stream>>>(p);
  return cuda_check(cudaGetLastError(), "fp32 profile launch");
}

int row_block(int d, int dtype) {
  if (dtype == SVG_FP32) return 4;
  return d == 128 ? ProfCfg<128>::ROWS : ProfCfg<64>::ROWS;
}

}  // namespace

bool profile_layout(int B, int H, int L, int d, int dtype, int S, ProfileLayout* out) {
  if (B < 1 || H < 1 || L < 1 || S < 1 || S > 128) return false;
  const int rb = row_block(d, dtype);
  ProfileLayout lay{};
  lay.S_pad = (S + rb - 1) / rb * rb;
  if (dtype == SVG_FP32) {
    lay.n_chunks = 1;
    lay.chunk = L;
  } else {
    // Aim for about four CTAs per SM over all heads and row blocks, with at
    // least four key tiles per chunk.
    const long long ctas_per_chunk = static_cast<long long>(B) * H * (lay.S_pad / rb);
    long long nch = (148LL * 4 + ctas_per_chunk - 1) / ctas_per_chunk;
    const long long max_nch = (L + 4 * kKT - 1) / (4 * kKT);
    if (nch > max_nch) nch = max_nch;
    if (nch < 1) nch = 1;
    long long chunk = (L + nch - 1) / nch;
    chunk = (chunk + kKT - 1) / kKT * kKT;
    lay.chunk = static_cast<int>(chunk);
    lay.n_chunks = static_cast<int>((L + chunk - 1) / chunk);
  }
  const size_t rows_total = static_cast<size_t>(B) * H * lay.n_chunks * 3 * lay.S_pad;
  lay.o_bytes = (rows_total * d * sizeof(float) + 255) / 256 * 256;
  lay.ml_bytes = (rows_total * 2 * sizeof(float) + 255) / 256 * 256;
  lay.total = lay.o_bytes + lay.ml_bytes;
  *out = lay;
  return true;
}

svg_status launch_profile(int B, int H, int N, int F, int d, int dtype, float scale, const void* q,
                          const void* k, const void* v, int a1, int a2, const int32_t* rows, int S,
                          float* mse, int8_t* label, void* ws, const ProfileLayout& lay,
                          cudaStream_t stream) {
  ProfParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.rows = rows;
  p.ws_o = static_cast<float*>(ws);
  p.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + lay.o_bytes);
  p.BH = B * H;
  p.L = N * F;
  p.N = N;
  p.F = F;
  p.S = S;
  p.S_pad = lay.S_pad;
  p.nch = lay.n_chunks;
  p.chunk = lay.chunk;
  p.a1 = a1;
  p.a2 = a2;
  p.sl2 = scale * 1.4426950408889634f;
  if (p.BH > 65535) return fail(SVG_ERR_UNSUPPORTED, "B*H = %d exceeds the grid limit", p.BH);
  svg_status st;
  if (dtype == SVG_BF16) {
    if (d == 64) st = launch_stage1_bf16<64>(p, stream);
    else if (d == 128) st = launch_stage1_bf16<128>(p, stream);
    else return fail(SVG_ERR_UNSUPPORTED, "bf16 profiling supports d in {64, 128}, got %d", d);
  } else {
    if (d == 32) st = launch_stage1_f32<32>(p, stream);
    else if (d == 64) st = launch_stage1_f32<64>(p, stream);
    else if (d == 128) st = launch_stage1_f32<128>(p, stream);
    else return fail(SVG_ERR_UNSUPPORTED, "fp32 profiling supports d in {32, 64, 128}, got %d", d);
  }
  if (st != SVG_OK) return st;
  profile_combine_kernel<<<p.BH, kCombineThreads, 0, stream>>>(p.ws_o, p.ws_ml, S, lay.S_pad, d, lay.n_chunks,
                                                                mse, label);
  return cuda_check(cudaGetLastError(), "profile combine launch");
}

}  // namespace svg
