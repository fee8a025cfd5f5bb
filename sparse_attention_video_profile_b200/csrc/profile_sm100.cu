// profile_sm100.cu -- stage 1 of online profiling on B200 tensor cores
// ("Sparse Video-Gen", Weakness 1 answer on online profiling: every step and
// layer, right before 3D attention; "Sparse VideoGen ...", Abstract: heads
// are classified spatial or temporal online).
//
// For the S sampled query rows of one head (padded to one 128-row tile) and
// one chunk of keys, computes three online-softmax attention states at once:
// unmasked (d), spatial |i_x - i_y| < a1 (s) and temporal |j_x - j_y| < a2
// (t).  Per 128-key tile:
//   S_k = Q K_k^T                     one tcgen05.mma group into TMEM
//   P_d, P_s, P_t (bf16) in shared memory -> O_v += P_v V_k, v = d, s, t
// The three variants share one softmax reference, the running max over all
// kept keys, so each key needs one exponential: P_s and P_t are P_d
// restricted to the spatial and temporal masks (the normalisation of each
// variant divides the reference out again).
// TMEM holds S and the three accumulators (all 512 columns at d = 128), so
// there is one S buffer; P goes to shared memory instead (three 32 KB
// K-major tiles, the A operands of the P V products), which frees S as soon
// as the softmax has read it.  The tensor cores then compute S_{k+1} while
// the softmax works on tile k, and the products of tile k follow; the
// softmax waits for the products of tile k-1 only before it overwrites P.
// The partial (max, sum, unnormalised output) triples of every row and
// variant go to the workspace; the combine kernels merge the chunks.
// TMEM: S [0,128), O_d [128,128+D), O_s [128+D,128+2D), O_t [128+2D,128+3D).
//
// Warps 0-7: two threads per sampled row, one per 64-key half of each tile
// (Q gather, masks, three softmaxes, epilogue); the halves exchange their
// maxima through shared memory once per tile.  Warp 8: TMA producer of K and
// V (the ring is short, so it also prefetches tiles further ahead into L2).
// Warp 9: MMA issuer.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace svg {

struct ProfSm100Params {
  CUtensorMap tm_k, tm_v;  // frame-major, laid out as hs
  const __nv_bfloat16* q;  // laid out as hs
  HeadStrides hs;
  const int32_t* rows;
  float* ws_o;   // [BH][nch][3][128][D]
  float* ws_ml;  // [BH][nch][3][128][2]  (max in log2 units, sum)
  int BH, L, N, F, S, nch, chunk;
  int kind[2], par[2];  // masks of the two restricted variants (ProfMaskKind)
  float sl2;
  float lazy_th;
  int* status;
  uint64_t wait_ns;
};

namespace {

// Masks of the restricted variants.
enum ProfMaskKind { kMaskFrameBand = 0, kMaskPositionBand = 1, kMaskWindow = 2, kMaskPrefix = 3, kMaskNone = 4 };

template <int D>
struct PCfg {
  static constexpr int HALVES = D / 64;
  static constexpr int HALF_BYTES = 128 * 128;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int P_BYTES = 128 * 128 * 2;  // one P tile: 128 rows x 128 keys, two 64-key halves
  static constexpr int NS = (D == 128) ? 2 : 6;
  static constexpr int PF = 4;                   // ring entries prefetched into L2 ahead of their load
  static constexpr int SMEM_P = TILE_BYTES + NS * TILE_BYTES;
  static constexpr int SMEM_BAR = SMEM_P + 3 * P_BYTES;
  static constexpr int SMEM_X = SMEM_BAR + 512;  // row-max exchange [2][2][128] + final sums [5][128] (fp32)
  static constexpr int SMEM_BYTES = SMEM_X + 5120 + 1024;
  // 10 warps: softmax 0-7 (warp w: rows 32 (w & 3) .. +31, key columns
  // 64 (w >> 2) .. +63 of each tile), TMA producer 8, MMA issuer 9.
  static constexpr int THREADS = 320;
  static constexpr uint32_t COL_S = 0;
  static constexpr uint32_t col_o(int v) { return 128u + D * v; }
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Prefetch of a 4D tile into L2 (no shared-memory destination, no completion).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// Pairs (of 8) of each half row's exponentials computed by the FMA-pipe
// polynomial instead of the MUFU ex2 unit.
#ifndef SVG_PROF_POLY_PAIRS
#define SVG_PROF_POLY_PAIRS 2
#endif
constexpr int kProfPolyPairs = SVG_PROF_POLY_PAIRS;

__device__ __forceinline__ bool warp_wait_p(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, limit);
  return __all_sync(0xffffffffu, ok);
}

// Sets bits [lo, hi) of a 64-bit mask held as two words (0 <= lo, hi <= 64).
__device__ __forceinline__ void set_range64(uint32_t (&m)[2], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int a = max(lo - 32 * w, 0), b = min(hi - 32 * w, 32);
    if (a < b) {
      const uint32_t hi_bits = (b >= 32) ? 0xFFFFFFFFu : ((1u << b) - 1u);
      m[w] |= hi_bits & ~((1u << a) - 1u);
    }
  }
}

// P_d of one half row: the weights e (already 0 for keys outside the chunk)
// as bf16 pairs, and the sum of the rounded weights of each 32-key word.
__device__ __forceinline__ void pack_plain(const float (&e)[64], uint32_t (&pk)[32], float (&wsum)[2]) {
#pragma unroll
  for (int wi = 0; wi < 2; ++wi) {
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = wi * 16 + c;
      const uint32_t pp = pack_bf16x2(e[2 * i], e[2 * i + 1]);
      if (c & 1) add_bf16x2_f32(a1, pp);
      else add_bf16x2_f32(a0, pp);
      pk[i] = pp;
    }
    wsum[wi] = (a0.x + a1.x) + (a0.y + a1.y);
  }
}

// A restricted variant's P of one half row: the P_d pairs with the halves
// whose mask bit is clear set to +0; returns the sum of its rounded weights.
// A 32-key word that the mask keeps whole reuses P_d's word sum, one it drops
// is zero.
__device__ __forceinline__ float pack_variant(const uint32_t (&pkd)[32], const float (&wsum)[2], const uint32_t (&m)[2],
                                              uint32_t (&pk)[32]) {
  float sum = 0.f;
#pragma unroll
  for (int wi = 0; wi < 2; ++wi) {
    const uint32_t mw = m[wi];
    if (mw == 0xFFFFFFFFu) {
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[wi * 16 + c] = pkd[wi * 16 + c];
      sum += wsum[wi];
    } else if (mw == 0u) {
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[wi * 16 + c] = 0u;
    } else {
      float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const int i = wi * 16 + c;
        const uint32_t lo = (mw >> (2 * c)) & 1u, hi = (mw >> (2 * c + 1)) & 1u;
        const uint32_t pp = pkd[i] & (((0u - lo) & 0x0000FFFFu) | ((0u - hi) << 16));
        if (c & 1) add_bf16x2_f32(a1, pp);
        else add_bf16x2_f32(a0, pp);
        pk[i] = pp;
      }
      sum += (a0.x + a1.x) + (a0.y + a1.y);
    }
  }
  return sum;
}

// Multiplies D/2 columns of an O accumulator (this thread's TMEM lane) by alpha.
template <int D>
__device__ __forceinline__ void rescale_o_half(uint32_t t_o, float alpha) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    uint32_t ov[32];
    tmem_ld32(t_o + c * 32, ov);
    tmem_wait_ld();
    reg_fence32(ov);
#pragma unroll
    for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
    tmem_st32(t_o + c * 32, ov);
  }
}

template <int D>
__global__ void __launch_bounds__(320, 1) profile_sm100_kernel(const __grid_constant__ ProfSm100Params p) {
  using C = PCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::TILE_BYTES;
  uint8_t* sP = smem + C::SMEM_P;               // [3] P_d, P_s, P_t (bf16, K-major, 128-byte swizzle)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* bar_q = bars;                       // 128 arrivals: Q gathered
  uint64_t* bar_full = bars + 1;                // [NS]
  uint64_t* bar_empty = bars + 1 + C::NS;       // [NS]
  uint64_t* bar_s = bars + 1 + 2 * C::NS;       // S_k ready (and every earlier product done)
  uint64_t* bar_sfree = bar_s + 1;              // 256 arrivals: S_k read, its columns free
  uint64_t* bar_p = bar_s + 2;                  // 256 arrivals: P_d, P_s, P_t of tile k written
  uint64_t* bar_pv = bar_s + 3;                 // the three P V products of tile k done
  uint64_t* bar_x = bar_s + 4;                  // [4] 64 arrivals: the two halves of 32 rows exchanged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_x + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xm = reinterpret_cast<float*>(smem + C::SMEM_X);  // [2 parity][2 half][128 rows] half-row maxima
  float* fin = xm + 512;                                    // [5][128] second half's sums and counts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int y_begin = chunk * p.chunk;
  const int y_end = min(p.L, y_begin + p.chunk);
  const int kt0 = y_begin / 128;
  const int nk = (y_end - y_begin + 127) / 128;

  if (threadIdx.x == 0) {
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) & SVG_DEV_TIMEOUT) ? 1 : 0;
    mbar_init(bar_q, 128);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_sfree, 256);
    mbar_init(bar_p, 256);
    mbar_init(bar_pv, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bar_x[q], 64);
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool run = (*abort_flag == 0);

  if (run && warp == 8 && lane == 0) {
    // ------------------------------------------------ TMA producer (K, V)
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    const int th = p.hs.tma_h(bh), tb = p.hs.tma_b(bh);
    // entry n of the ring: K_0, then K_{k+1} ahead of V_k (the order the MMA
    // warp consumes them): K_0, K_1, V_0, K_2, V_1, ..., K_{nk-1}, V_{nk-2}, V_{nk-1}
    auto entry_tile = [&](int n, bool& is_v) {
      if (n == 0) {
        is_v = false;
        return 0;
      }
      if ((n & 1) && (n + 1) / 2 < nk) {
        is_v = false;
        return (n + 1) / 2;
      }
      is_v = true;
      return (n & 1) ? nk - 1 : n / 2 - 1;
    };
    auto prefetch = [&](int n) {
      bool is_v;
      const int t = entry_tile(n, is_v);
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h)
        tma_prefetch_l2_4d(is_v ? &p.tm_v : &p.tm_k, h * 64, (kt0 + t) * 128, th, tb);
    };
    for (int n = 0; n < min(C::PF, 2 * nk); ++n) prefetch(n);
    for (int n = 0; n < 2 * nk; ++n) {
      const int slot = n % C::NS;
      if (n + C::PF < 2 * nk) prefetch(n + C::PF);  // on its way to L2 while n waits for its slot
      if (!mbar_wait(&bar_empty[slot], ((n / C::NS) & 1) ^ 1, p.wait_ns)) {
        *abort_flag = 1;
        atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
        break;
      }
      bool is_v;
      const int t = entry_tile(n, is_v);
      in_range((kt0 + t) * 128, p.L, p.status);
      mbar_arrive_expect_tx(&bar_full[slot], C::TILE_BYTES);
#pragma unroll
      for (int h = 0; h < C::HALVES; ++h)
        tma_load_4d(sRing + slot * C::TILE_BYTES + h * C::HALF_BYTES, is_v ? &p.tm_v : &p.tm_k, &bar_full[slot],
                    h * 64, (kt0 + t) * 128, th, tb);
    }
  } else if (run && warp == 9) {
    // ------------------------------------------------ MMA issuer
    // The whole warp runs the loop with warp-uniform operands; one elected
    // lane issues each tcgen05 instruction.
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t ring_base = smem_u32(sRing);
    const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dk = smem_desc_sw128(ring_base, 16, 1024);
    const uint64_t dv = smem_desc_sw128(ring_base, C::HALF_BYTES, 1024);
    const uint64_t dp = smem_desc_sw128(smem_u32(sP), 16, 1024);
    // O_v += P_v V: A = P_v (K-major in shared memory), B = V (MN-major)
    auto pv = [&](int v, int slot, bool acc) {
      const uint64_t a = dp + static_cast<uint64_t>((v * C::P_BYTES) >> 4);
      const uint64_t b = dv + static_cast<uint64_t>((slot * C::TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t aoff = static_cast<uint64_t>(((kk >> 2) * C::HALF_BYTES + (kk & 3) * 32) >> 4);
        umma_ss_warp(tmem + C::col_o(v), a + aoff, b + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv,
                     (acc || kk > 0) ? 1u : 0u);
      }
    };
    // S_k = Q K_k^T into the S columns
    auto qk = [&](int slot) {
      const uint64_t b = dk + static_cast<uint64_t>((slot * C::TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::HALF_BYTES + (kk & 3) * 32) >> 4);
        umma_ss_warp(tmem + C::COL_S, dq + off, b + off, idesc_qk, kk > 0 ? 1u : 0u);
      }
      umma_commit_warp(bar_s);
      umma_commit_warp(&bar_empty[slot]);
    };
    // Ring entries (the producer's order): K_0 is entry 0, K_{k+1} entry
    // 2k + 1, V_k entry 2k + 2 (the last V entry 2 nk - 1).  S_{k+1} goes in
    // as soon as the softmax has read S_k, ahead of the products of tile k.
    bool ok = warp_wait_p(bar_q, 0, p.wait_ns) && warp_wait_p(&bar_full[0], 0, p.wait_ns);
    if (ok) {
      tc_fence_after();
      qk(0);
    }
    for (int k = 0; ok && k < nk; ++k) {
      if (k + 1 < nk) {
        const int nK = 2 * k + 1, slotK = nK % C::NS;
        ok = warp_wait_p(bar_sfree, k & 1, p.wait_ns) && warp_wait_p(&bar_full[slotK], (nK / C::NS) & 1, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        qk(slotK);
      }
      const int nV = (k + 1 < nk) ? 2 * k + 2 : 2 * nk - 1, slotV = nV % C::NS;
      ok = warp_wait_p(bar_p, k & 1, p.wait_ns) && warp_wait_p(&bar_full[slotV], (nV / C::NS) & 1, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      pv(0, slotV, k > 0);  // O_d += P_d V
      pv(1, slotV, k > 0);  // O_s += P_s V
      pv(2, slotV, k > 0);  // O_t += P_t V
      umma_commit_warp(bar_pv);
      umma_commit_warp(&bar_empty[slotV]);
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
    }
  } else if (run && warp < 8) {
    // ------------------------------------------------ rows: gather, softmax, epilogue
    // Two threads per sampled row: half h handles key columns [64 h, 64 h + 64)
    // of every tile.  The halves exchange their maxima once per tile so both
    // scale their weights by the same reference.
    const int q = warp & 3, h = warp >> 2;
    const int r = q * 32 + lane;  // row of the tile = sampled-row index (padded)
    in_range(p.rows[min(r, p.S - 1)], p.L, p.status);  // checked build: a sampled row outside [0, L) is reported
    const int x = min(max(p.rows[min(r, p.S - 1)], 0), p.L - 1);
    if (h == 0) {
      // gather Q row x into the 128-byte-swizzled K-major tile layout
      const uint4* src = reinterpret_cast<const uint4*>(p.q + p.hs.head(bh) + x * p.hs.sl);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        const uint4 val = __ldg(src + c);
        const int hh = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(sQ + hh * C::HALF_BYTES + r * 128 + ((cc ^ (r & 7)) << 4)) = val;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(bar_q);
    }
    const int ir = x / p.F, jr = x - (x / p.F) * p.F;
    // each restricted variant keeps one key interval of this row, except the
    // in-frame-position band, which keeps a window in every frame
    int lo_v[2], hi_v[2];
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int kind = p.kind[v], a = p.par[v];
      lo_v[v] = 0;
      hi_v[v] = 0;
      if (kind == kMaskFrameBand) {
        lo_v[v] = max(0, (ir - a + 1) * p.F);
        hi_v[v] = min(p.L, (ir + a) * p.F);
      } else if (kind == kMaskWindow) {
        lo_v[v] = max(0, x - a);
        hi_v[v] = min(p.L, x + a + 1);
      } else if (kind == kMaskPrefix) {
        hi_v[v] = min(p.L, a);
      }
    }
    const uint32_t lane_bits = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tS = tmem + lane_bits + C::COL_S;
    const uint32_t tO = tmem + lane_bits + h * (D / 2);  // + col_o(v): this half's output columns
    const float sl2 = p.sl2;
    // One softmax reference (the running max over all kept keys of the row)
    // serves the three variants: P_s and P_t are P_d restricted to their masks.
    float m_ref = -INFINITY, l_d = 0.f, l_s = 0.f, l_t = 0.f;
    // in-frame position of this half's first key, carried from tile to tile
    // (one division here instead of one per tile)
    int j0h = ((kt0 * 128 + h * 64) % p.F);
    int inband_s = 0, inband_t = 0;
    bool ok = true;
    for (int k = 0; k < nk; ++k) {
      if (!warp_wait_p(bar_s, k & 1, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tS + h * 64, sr[0]);
      tmem_ld32(tS + h * 64 + 32, sr[1]);
      tmem_wait_ld();
      reg_fence32(sr[0]);
      reg_fence32(sr[1]);
      tc_fence_before();
      mbar_arrive(bar_sfree);  // S_{k+1} may overwrite the columns
      float s[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c >> 5][c & 31]);

      const int kbase = (kt0 + k) * 128 + h * 64;  // key of this half's first column
      const int nv = min(64, y_end - kbase);        // keys of the chunk in this half (may be <= 0)
      // Key masks of the restricted variants: one key interval or, for the
      // in-frame-position band, |j - j_r| < a within each frame segment.
      uint32_t ms[2] = {0u, 0u}, mt[2] = {0u, 0u};
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        uint32_t(&mv)[2] = v ? mt : ms;
        if (p.kind[v] == kMaskPositionBand) {
          const int a = p.par[v];
          int c = 0;
          int j0 = j0h;
          while (c < nv) {  // one frame segment per pass: keys c .. c + (F - j0) - 1
            const int seg_end = min(nv, c + (p.F - j0));
            const int lo = max(c, c + (jr - a + 1 - j0));
            const int hi = min(seg_end, c + (jr + a - j0));
            if (lo < hi) set_range64(mv, lo, hi);
            c = seg_end;
            j0 = 0;
          }
        } else {
          set_range64(mv, max(lo_v[v] - kbase, 0), min(hi_v[v] - kbase, nv));
        }
      }
      j0h += 128;  // the next tile's first key of this half
      if (j0h >= p.F) j0h = (p.F >= 128) ? j0h - p.F : j0h % p.F;
      // keys past the chunk end get weight 0 in every variant
      if (nv < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= nv) s[c] = -INFINITY;
      }
      float m0 = fmaxf(s[0], s[1]), m1 = fmaxf(s[2], s[3]), m2 = fmaxf(s[4], s[5]), m3 = fmaxf(s[6], s[7]);
#pragma unroll
      for (int c = 8; c < 64; c += 8) {
        m0 = fmax3f(m0, s[c], s[c + 1]);
        m1 = fmax3f(m1, s[c + 2], s[c + 3]);
        m2 = fmax3f(m2, s[c + 4], s[c + 5]);
        m3 = fmax3f(m3, s[c + 6], s[c + 7]);
      }
      const float mh = fmaxf(fmax3f(m0, m1, m2), m3);
      // The row's maximum over the whole tile, from both halves.
      float* xk = xm + (k & 1) * 256;
      xk[h * 128 + r] = mh;
      mbar_arrive(&bar_x[q]);
      if (!warp_wait_p(&bar_x[q], k & 1, p.wait_ns)) {
        ok = false;
        break;
      }
      const float m_new = fmax3f(m_ref, mh, xk[(h ^ 1) * 128 + r]);
      float alpha = 1.f;
      bool resc = false;
      if (m_new > m_ref + p.lazy_th) {
        alpha = ex2_approx((m_ref - m_new) * sl2);
        m_ref = m_new;
        resc = true;
      }
      const float nb = (m_ref == -INFINITY) ? 0.f : -m_ref * sl2;
      {
        const float2 sl2x2 = make_float2(sl2, sl2), nb2 = make_float2(nb, nb);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 xx = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sl2x2, nb2);
          float2 e;
          if ((c & 7) < kProfPolyPairs) {
            // FMA-pipe polynomial (both halves of a row share one MUFU unit);
            // it clamps its argument, so weights that underflow, masked keys
            // and keys past the chunk end included, are set to 0 as ex2 does
            e = exp2_poly2(xx);
            e.x = xx.x < -126.f ? 0.f : e.x;
            e.y = xx.y < -126.f ? 0.f : e.y;
          } else {
            e.x = ex2_approx(xx.x);
            e.y = ex2_approx(xx.y);
          }
          s[2 * c] = e.x;  // s now holds the weights e
          s[2 * c + 1] = e.y;
        }
      }
      inband_s += __popc(ms[0]) + __popc(ms[1]);
      inband_t += __popc(mt[0]) + __popc(mt[1]);
      uint32_t pkd[32], pk[32];
      float wsum[2];
      pack_plain(s, pkd, wsum);
      l_d = l_d * alpha + (wsum[0] + wsum[1]);
      // the products of tile k-1 read P and add into O: wait for them before
      // overwriting P or rescaling O (bar_s of this tile already covers the
      // products of tile k-2, so the barrier is never two phases behind)
      if (k > 0) {
        if (!warp_wait_p(bar_pv, (k - 1) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // this half row = 64 keys = one 128-byte row of a swizzled 64-key block
      uint8_t* prow = sP + h * C::HALF_BYTES + r * 128;
      auto store_p = [&](int v, const uint32_t(&w)[32]) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(prow + v * C::P_BYTES + ((c ^ (r & 7)) << 4)) =
              make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      };
      store_p(0, pkd);
      l_s = l_s * alpha + pack_variant(pkd, wsum, ms, pk);
      store_p(1, pk);
      l_t = l_t * alpha + pack_variant(pkd, wsum, mt, pk);
      store_p(2, pk);
      // both halves of a row take the same decision (same reference)
      if (k > 0 && __any_sync(0xffffffffu, resc)) {
        rescale_o_half<D>(tO + C::col_o(0), alpha);
        rescale_o_half<D>(tO + C::col_o(1), alpha);
        rescale_o_half<D>(tO + C::col_o(2), alpha);
        tmem_wait_st();
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // P visible to the tensor cores
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    // the first half of each row collects the second half's sums and counts
    if (ok) {
      if (h == 1) {
        fin[r] = l_d;
        fin[128 + r] = l_s;
        fin[256 + r] = l_t;
        fin[384 + r] = __int_as_float(inband_s);
        fin[512 + r] = __int_as_float(inband_t);
      }
      mbar_arrive(&bar_x[q]);
      ok = warp_wait_p(&bar_x[q], nk & 1, p.wait_ns);
    }
    if (ok && h == 0) {
      l_d += fin[r];
      l_s += fin[128 + r];
      l_t += fin[256 + r];
      inband_s += __float_as_int(fin[384 + r]);
      inband_t += __float_as_int(fin[512 + r]);
      // Kept keys whose weights all underflowed relative to the shared
      // reference (in-band logits more than ~126 / (scale log2 e) below the
      // row max): report it rather than return a wrong label.
      if ((inband_s > 0 && !(l_s > 0.f)) || (inband_t > 0 && !(l_t > 0.f))) atomicOr(p.status, SVG_DEV_RANGE);
    }
    if (ok && warp_wait_p(bar_pv, (nk - 1) & 1, p.wait_ns)) {
      tc_fence_after();
#pragma unroll
      for (int v = 0; v < 3; ++v) {
        const size_t base = ((static_cast<size_t>(bh) * p.nch + chunk) * 3 + v) * 128 + r;
        // checked build: a slot outside the workspace is reported and its stores
        // skipped (the tensor-memory loads below are warp-collective and stay)
        const bool store_ok =
            in_range(static_cast<long long>(base), static_cast<long long>(p.BH) * p.nch * 3 * 128, p.status);
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (store_ok ? base : 0) * D + h * (D / 2));
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t ov[32];
          __syncwarp();
          tmem_ld32(tO + C::col_o(v) + c * 32, ov);
          tmem_wait_ld();
          reg_fence32(ov);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (store_ok)
              dst[c * 8 + e] = make_float4(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]),
                                           __uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
        }
        if (h == 0 && store_ok) {
          const float lv = (v == 0) ? l_d : (v == 1 ? l_s : l_t);
          const int nin = (v == 0) ? 1 : (v == 1 ? inband_s : inband_t);
          // max in log2 units; a variant with no kept key in this chunk has none
          p.ws_ml[base * 2 + 0] = (m_ref == -INFINITY || nin == 0) ? -INFINITY : m_ref * sl2;
          p.ws_ml[base * 2 + 1] = lv;
        }
      }
    } else {
      *abort_flag = 1;
      atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

template <int D>
svg_status launch_profile_sm100_d(ProfSm100Params& p, const void* k, const void* v, cudaStream_t stream) {
  using C = PCfg<D>;
  svg_status st;
  if ((st = make_tile_map_bf16(&p.tm_k, k, p.hs, p.L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_v, v, p.hs, p.L, D)) != SVG_OK) return st;
  cudaError_t e = cudaFuncSetAttribute(profile_sm100_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute(profile smem)");
  profile_sm100_kernel<D><<<dim3(p.nch, p.BH), C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cuda_check(cudaGetLastError(), "profile launch");
}

svg_status launch_profile_sm100(int BH, int N, int F, int d, float scale, const void* q, const void* k,
                                const void* v, const HeadStrides& hs, const int (&kind)[2], const int (&par)[2], const int32_t* rows, int S,
                                float* ws_o, float* ws_ml, int nch, int chunk, int* status, cudaStream_t stream) {
  ProfSm100Params p;
  memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.hs = hs;
  p.rows = rows;
  p.ws_o = ws_o;
  p.ws_ml = ws_ml;
  p.BH = BH;
  p.L = N * F;
  p.N = N;
  p.F = F;
  p.S = S;
  p.nch = nch;
  p.chunk = chunk;
  for (int i = 0; i < 2; ++i) {
    p.kind[i] = kind[i];
    p.par[i] = par[i];
  }
  p.sl2 = scale * 1.4426950408889634f;
  p.lazy_th = 8.0f / p.sl2;
  p.status = status;
  p.wait_ns = kDefaultWaitNs;
  if (d == 64) return launch_profile_sm100_d<64>(p, k, v, stream);
  if (d == 128) return launch_profile_sm100_d<128>(p, k, v, stream);
  return fail(SVG_ERR_UNSUPPORTED, "bf16 profiling supports d in {64, 128}, got %d", d);
}

}  // namespace svg
