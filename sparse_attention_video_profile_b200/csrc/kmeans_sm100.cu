// kmeans_sm100.cu -- k-means of a head's Q or K rows, the clustering step of
// SVG2-style sparse attention (SVG2 explainer, 2.A: Q and K are clustered
// independently by k-means before attention).
//
// Lloyd's algorithm from the rows floor(c L / C):
//   assign  every row to its nearest centroid: argmin_c ||m_c||^2 - 2 x . m_c
//           with m_c the centroid rounded to bf16 (the tensor cores multiply
//           bf16) and ||m_c||^2 taken of that rounded centroid in fp32; ties
//           go to the lower index.  kmeans_assign_kernel is a tcgen05 GEMM
//           (M = 128 rows, N = up to 256 centroids per MMA, K = d) with the
//           argmin fused into its epilogue: the centroids stay in shared
//           memory for the whole CTA, row tiles stream through a 2-slot TMA
//           ring, and the score accumulator alternates between two 256-column
//           TMEM slots so the epilogue of one overlaps the MMAs of the next.
//           The argmin runs on eight warps, two threads per row, each
//           scanning half of every slot's columns; the halves compare their
//           results once per row tile through shared memory.
//   update  each centroid to the mean of its rows: the counting sort by
//           cluster (svg2_sort), then eight warps per cluster summing its
//           rows in fp32 in a fixed order (deterministic); an empty cluster
//           keeps its centroid.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace svg {

namespace {

constexpr int kKmThreads = 320;  // warps 0-7 epilogue (two threads per row), 8 TMA, 9 MMA
constexpr int kKmSlotCols = 256;

struct KmParams {
  CUtensorMap tm_x;  // rows of x, laid out as xs, box 64 x 128
  CUtensorMap tm_c;  // bf16 centroids: [BH, C, D], box 64 x 128
  HeadStrides xs;
  const float* norm;  // [BH][C] ||bf16 centroid||^2
  int32_t* assign;    // [BH][L]
  int L, C, C_pad, nch, tiles, tiles_per_cta;
  int slot_cols;  // TMEM columns per score slot: min(256, C_pad); 2 slots allocated
  int* status;
  uint64_t wait_ns;
};

template <int D>
struct KmCfg {
  static constexpr int HALVES = D / 64;
  static constexpr int TILE_BYTES = 128 * D * 2;   // one row tile
  static constexpr int HALF_BYTES = 128 * 128;     // 128 rows x 128 bytes
};

__device__ __forceinline__ bool km_warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, limit);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(kKmThreads, 1) kmeans_assign_kernel(const __grid_constant__ KmParams p) {
  using K = KmCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sC = smem;                                                       // centroids, C_pad rows per 64-col half
  uint8_t* sX = smem + static_cast<size_t>(p.C_pad) * 128 * K::HALVES;      // 2 row tiles
  float* sNorm = reinterpret_cast<float*>(sX + 2 * K::TILE_BYTES);           // [C_pad]
  float* xbest = sNorm + p.C_pad;                                           // [2 parity][128 rows] second half's minimum
  int* xbi = reinterpret_cast<int*>(xbest + 256);                           // [2][128] and its column
  uint64_t* bars = reinterpret_cast<uint64_t*>(xbi + 256);
  uint64_t* bar_c = bars;              // centroids loaded
  uint64_t* bar_xfull = bars + 1;      // [2]
  uint64_t* bar_xempty = bars + 3;     // [2]
  uint64_t* bar_s = bars + 5;          // [2] scores of a TMEM slot ready
  uint64_t* bar_free = bars + 7;       // [2] epilogue done with a TMEM slot (256 arrivals)
  uint64_t* bar_x = bars + 9;          // [4] the two halves of 32 rows compared (64 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int t_begin = blockIdx.x * p.tiles_per_cta;
  const int t_end = min(p.tiles, t_begin + p.tiles_per_cta);
  const int nt = t_end > t_begin ? t_end - t_begin : 0;

  if (threadIdx.x == 0) {
    mbar_init(bar_c, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_xfull[i], 1);
      mbar_init(&bar_xempty[i], 1);
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_free[i], 256);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&bar_x[q], 64);
    fence_barrier_init();
  }
  // padding centroids score +inf, so they never win the argmin
  for (int c = threadIdx.x; c < p.C_pad; c += kKmThreads)
    sNorm[c] = c < p.C ? p.norm[static_cast<size_t>(bh) * p.C + c] : INFINITY;
  if (warp == 9) {
    tmem_alloc(tmem_slot, 2 * p.slot_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (nt > 0 && warp == 8 && lane == 0) {
    // ---------------------------------------------- TMA producer
    tma_prefetch_desc(&p.tm_c);
    tma_prefetch_desc(&p.tm_x);
    mbar_arrive_expect_tx(bar_c, static_cast<uint32_t>(p.C_pad) * D * 2);
    for (int r = 0; r < p.C_pad; r += 128)
#pragma unroll
      for (int h = 0; h < K::HALVES; ++h)
        tma_load_4d(sC + static_cast<size_t>(h) * p.C_pad * 128 + static_cast<size_t>(r) * 128, &p.tm_c, bar_c, h * 64,
                    r, bh, 0);
    const int th = p.xs.tma_h(bh), tb = p.xs.tma_b(bh);
    for (int i = 0; i < nt; ++i) {
      const int s = i & 1;
      if (!mbar_wait(&bar_xempty[s], ((i >> 1) & 1) ^ 1, p.wait_ns)) {
        atomicOr(p.status, SVG_DEV_TIMEOUT);
        break;
      }
      mbar_arrive_expect_tx(&bar_xfull[s], K::TILE_BYTES);
#pragma unroll
      for (int h = 0; h < K::HALVES; ++h)
        tma_load_4d(sX + s * K::TILE_BYTES + h * K::HALF_BYTES, &p.tm_x, &bar_xfull[s], h * 64, (t_begin + i) * 128, th,
                    tb);
    }
  } else if (nt > 0 && warp == 9) {
    // ---------------------------------------------- MMA issuer (whole warp, elected lane issues)
    const uint64_t dc = smem_desc_sw128(smem_u32(sC), 16, 1024);
    const uint64_t dx = smem_desc_sw128(smem_u32(sX), 16, 1024);
    bool ok = km_warp_wait(bar_c, 0, p.wait_ns);
    for (int i = 0; ok && i < nt; ++i) {
      const int xs = i & 1;
      ok = km_warp_wait(&bar_xfull[xs], (i >> 1) & 1, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      for (int j = 0; j < p.nch; ++j) {
        const int u = i * p.nch + j, s = u & 1;
        ok = km_warp_wait(&bar_free[s], ((u >> 1) & 1) ^ 1, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        const int width = min(kKmSlotCols, p.C_pad - j * kKmSlotCols);  // a multiple of 128
        const uint32_t idesc = idesc_bf16_f32(128, width, 0, 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a =
              dx + static_cast<uint64_t>((xs * K::TILE_BYTES + (kk >> 2) * K::HALF_BYTES + (kk & 3) * 32) >> 4);
          const uint64_t b = dc + static_cast<uint64_t>(
                                      ((kk >> 2) * static_cast<size_t>(p.C_pad) * 128 +
                                       static_cast<size_t>(j) * kKmSlotCols * 128 + (kk & 3) * 32) >> 4);
          umma_ss_warp(tmem + s * p.slot_cols, a, b, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit_warp(&bar_s[s]);
      }
      if (!ok) break;
      umma_commit_warp(&bar_xempty[xs]);  // the row tile is free once its MMAs are done
    }
    if (!ok && lane == 0) atomicOr(p.status, SVG_DEV_TIMEOUT);
  } else if (nt > 0 && warp < 8) {
    // ---------------------------------------------- epilogue: argmin per row
    // warps q and q + 4 share rows 32 q .. 32 q + 31: half hh scans columns
    // [hh w/2, (hh + 1) w/2) of every slot of width w
    const int q = warp & 3, hh = warp >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(q * 32) << 16;
    for (int i = 0; i < nt; ++i) {
      float best = INFINITY;
      int bi = 0;
      bool ok = true;
      for (int j = 0; j < p.nch; ++j) {
        const int u = i * p.nch + j, s = u & 1;
        if (!km_warp_wait(&bar_s[s], (u >> 1) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int width = min(kKmSlotCols, p.C_pad - j * kKmSlotCols);
        const int c_begin = hh * (width / 2), c_end = c_begin + width / 2;  // multiples of 64
        const uint32_t ts = tmem + lane_bits + s * p.slot_cols;
        // 32 columns at a time, the next load in flight while this one is reduced
        uint32_t v[2][32];
        tmem_ld32(ts + c_begin, v[0]);
        tmem_wait_ld();
        reg_fence32(v[0]);
        for (int c0 = c_begin; c0 < c_end; c0 += 64) {
          tmem_ld32(ts + c0 + 32, v[1]);  // width is a multiple of 128
          const float* nrm = sNorm + j * kKmSlotCols + c0;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float score = fmaf(-2.f, __uint_as_float(v[0][e]), nrm[e]);
            if (score < best) {  // ascending columns: ties keep the lower index
              best = score;
              bi = j * kKmSlotCols + c0 + e;
            }
          }
          tmem_wait_ld();
          reg_fence32(v[1]);
          if (c0 + 64 < c_end) tmem_ld32(ts + c0 + 64, v[0]);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float score = fmaf(-2.f, __uint_as_float(v[1][e]), nrm[32 + e]);
            if (score < best) {
              best = score;
              bi = j * kKmSlotCols + c0 + 32 + e;
            }
          }
          if (c0 + 64 < c_end) {
            tmem_wait_ld();
            reg_fence32(v[0]);
          }
        }
        tc_fence_before();
        mbar_arrive(&bar_free[s]);
      }
      if (ok) {
        // the second half hands its minimum to the first; ties go to the
        // lower column, wherever it was found
        if (hh == 1) {
          xbest[(i & 1) * 128 + r] = best;
          xbi[(i & 1) * 128 + r] = bi;
        }
        mbar_arrive(&bar_x[q]);
        ok = km_warp_wait(&bar_x[q], i & 1, p.wait_ns);
      }
      if (!ok) {
        if (lane == 0) atomicOr(p.status, SVG_DEV_TIMEOUT);
        break;
      }
      if (hh == 0) {
        const float b1 = xbest[(i & 1) * 128 + r];
        const int i1 = xbi[(i & 1) * 128 + r];
        if (b1 < best || (b1 == best && i1 < bi)) {
          best = b1;
          bi = i1;
        }
        const int row = (t_begin + i) * 128 + r;
        // checked build: the chosen centroid is one of the C real ones
        if (row < p.L && in_range(bi, p.C, p.status)) p.assign[static_cast<size_t>(bh) * p.L + row] = bi;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * p.slot_cols);
  }
}

// Centroids of the rows floor(c L / C) (fp32, bf16 copy, norm of the copy).
template <int D>
__global__ void __launch_bounds__(32) kmeans_init_kernel(const __nv_bfloat16* __restrict__ x, const HeadStrides xs,
                                                         int L, int C, float* __restrict__ mu,
                                                         __nv_bfloat16* __restrict__ mu_b, float* __restrict__ norm) {
  constexpr int PER = D / 32;
  const int c = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
  const long long r = static_cast<long long>(c) * L / C;
  const __nv_bfloat16* xr = x + xs.head(bh) + r * xs.sl;
  const size_t o = (static_cast<size_t>(bh) * C + c) * D;
  float n2 = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const __nv_bfloat16 b = xr[e * 32 + lane];
    const float f = __bfloat162float(b);
    mu[o + e * 32 + lane] = f;
    mu_b[o + e * 32 + lane] = b;
    n2 = fmaf(f, f, n2);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, off);
  if (lane == 0) norm[static_cast<size_t>(bh) * C + c] = n2;
}

// Each centroid becomes the mean of its rows (read through the permutation);
// an empty cluster keeps its centroid.  kUpdWarps warps per cluster: warp w
// sums rows w, w + W, w + 2W, ... (two rows in flight), and the partial sums
// are added in warp order: a fixed order, so the result is deterministic.
constexpr int kUpdWarps = 8;

template <int D>
__global__ void __launch_bounds__(kUpdWarps * 32) kmeans_update_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const HeadStrides xs,
                                                            const int32_t* __restrict__ perm,
                                                            const int32_t* __restrict__ off, int L, int C,
                                                            float* __restrict__ mu, __nv_bfloat16* __restrict__ mu_b,
                                                            float* __restrict__ norm) {
  constexpr int PER = D / 32;
  __shared__ float part[kUpdWarps][D];
  const int c = blockIdx.x, bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* o = off + static_cast<size_t>(bh) * (C + 1);
  const int r0 = o[c], r1 = o[c + 1];
  const size_t mo = (static_cast<size_t>(bh) * C + c) * D;
  float s[PER], t[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) s[e] = t[e] = 0.f;
  const __nv_bfloat16* xh = x + xs.head(bh);
  const long long sl = xs.sl;
  const int32_t* pm = perm + static_cast<size_t>(bh) * L;
  int r = r0 + warp;
  for (; r + kUpdWarps < r1; r += 2 * kUpdWarps) {  // two independent rows per step
    const __nv_bfloat16* xa = xh + pm[r] * sl;
    const __nv_bfloat16* xb = xh + pm[r + kUpdWarps] * sl;
    __nv_bfloat16 va[PER], vb[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      va[e] = xa[e * 32 + lane];
      vb[e] = xb[e * 32 + lane];
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      s[e] += __bfloat162float(va[e]);
      t[e] += __bfloat162float(vb[e]);
    }
  }
  if (r < r1) {
    const __nv_bfloat16* xa = xh + pm[r] * sl;
#pragma unroll
    for (int e = 0; e < PER; ++e) s[e] += __bfloat162float(xa[e * 32 + lane]);
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) part[warp][e * 32 + lane] = s[e] + t[e];
  __syncthreads();
  if (warp != 0) return;
  float m[PER];
  if (r1 > r0) {
    const float inv = 1.f / static_cast<float>(r1 - r0);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int col = e * 32 + lane;
      float acc = part[0][col];
#pragma unroll
      for (int w = 1; w < kUpdWarps; ++w) acc += part[w][col];
      m[e] = acc * inv;
      mu[mo + col] = m[e];
    }
  } else {
#pragma unroll
    for (int e = 0; e < PER; ++e) m[e] = mu[mo + e * 32 + lane];
  }
  float n2 = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const __nv_bfloat16 b = __float2bfloat16_rn(m[e]);
    mu_b[mo + e * 32 + lane] = b;
    const float f = __bfloat162float(b);
    n2 = fmaf(f, f, n2);
  }
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, sh);
  if (lane == 0) norm[static_cast<size_t>(bh) * C + c] = n2;
}

template <int D>
svg_status launch_assign(const void* x, const HeadStrides& xs, const __nv_bfloat16* mu_b, const float* norm, int BH,
                         int L, int C, int32_t* assign, int* status, cudaStream_t stream) {
  using K = KmCfg<D>;
  KmParams p;
  memset(&p, 0, sizeof(p));
  svg_status st;
  p.xs = xs;
  if ((st = make_tile_map_bf16(&p.tm_x, x, xs, L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_c, mu_b, dense_strides(1, BH, C, D), C, D)) != SVG_OK) return st;
  p.norm = norm;
  p.assign = assign;
  p.L = L;
  p.C = C;
  p.C_pad = (C + 127) / 128 * 128;
  p.nch = (p.C_pad + kKmSlotCols - 1) / kKmSlotCols;
  p.slot_cols = p.C_pad < kKmSlotCols ? p.C_pad : kKmSlotCols;
  p.tiles = (L + 127) / 128;
  int per_head = 148 / BH;
  if (per_head < 1) per_head = 1;
  if (per_head > p.tiles) per_head = p.tiles;
  p.tiles_per_cta = (p.tiles + per_head - 1) / per_head;
  const int nx = (p.tiles + p.tiles_per_cta - 1) / p.tiles_per_cta;
  p.status = status;
  p.wait_ns = 1000000000ull;
  const size_t smem = 1024 + static_cast<size_t>(p.C_pad) * 128 * K::HALVES + 2 * K::TILE_BYTES +
                      static_cast<size_t>(p.C_pad) * 4 + 2048 + 128;
  if (smem > 227 * 1024) return fail(SVG_ERR_UNSUPPORTED, "k-means with C = %d does not fit shared memory", C);
  cudaError_t e = cudaFuncSetAttribute(kmeans_assign_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute(k-means smem)");
  kmeans_assign_kernel<D><<<dim3(nx, BH), kKmThreads, smem, stream>>>(p);
  return cuda_check(cudaGetLastError(), "k-means assign launch");
}

}  // namespace

size_t kmeans_workspace_bytes(int BH, int L, int C, int d) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  const int nblk = (L + 2047) / 2048;
  return al(static_cast<size_t>(BH) * C * d * 2)       // bf16 centroids
         + al(static_cast<size_t>(BH) * C * 4)          // norms
         + al(static_cast<size_t>(BH) * C * nblk * 4)   // sort histogram
         + 2 * al(static_cast<size_t>(BH) * L * 4)      // permutation, clusters in permuted order
         + al(static_cast<size_t>(BH) * (C + 1) * 4);   // offsets
}

svg_status launch_kmeans(const void* x, const HeadStrides& xs, int BH, int L, int C, int d, int iters, int32_t* assign,
                         float* mu, void* workspace, int* status, cudaStream_t stream) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  const int nblk = (L + 2047) / 2048;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* mu_b = reinterpret_cast<__nv_bfloat16*>(w);
  w += al(static_cast<size_t>(BH) * C * d * 2);
  float* norm = reinterpret_cast<float*>(w);
  w += al(static_cast<size_t>(BH) * C * 4);
  int32_t* hist = reinterpret_cast<int32_t*>(w);
  w += al(static_cast<size_t>(BH) * C * nblk * 4);
  int32_t* perm = reinterpret_cast<int32_t*>(w);
  w += al(static_cast<size_t>(BH) * L * 4);
  int32_t* cid = reinterpret_cast<int32_t*>(w);
  w += al(static_cast<size_t>(BH) * L * 4);
  int32_t* off = reinterpret_cast<int32_t*>(w);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (d == 128)
    kmeans_init_kernel<128><<<dim3(C, BH), 32, 0, stream>>>(xb, xs, L, C, mu, mu_b, norm);
  else
    kmeans_init_kernel<64><<<dim3(C, BH), 32, 0, stream>>>(xb, xs, L, C, mu, mu_b, norm);
  svg_status st = cuda_check(cudaGetLastError(), "k-means init launch");
  for (int it = 0; st == SVG_OK && it < iters; ++it) {
    st = d == 128 ? launch_assign<128>(x, xs, mu_b, norm, BH, L, C, assign, status, stream)
                  : launch_assign<64>(x, xs, mu_b, norm, BH, L, C, assign, status, stream);
    if (st != SVG_OK) break;
    if ((st = svg2_sort(assign, BH, L, C, nblk, hist, perm, cid, off, status, stream)) != SVG_OK) break;
    if (d == 128)
      kmeans_update_kernel<128><<<dim3(C, BH), kUpdWarps * 32, 0, stream>>>(xb, xs, perm, off, L, C, mu, mu_b, norm);
    else
      kmeans_update_kernel<64><<<dim3(C, BH), kUpdWarps * 32, 0, stream>>>(xb, xs, perm, off, L, C, mu, mu_b, norm);
    st = cuda_check(cudaGetLastError(), "k-means update launch");
  }
  return st;
}

}  // namespace svg
