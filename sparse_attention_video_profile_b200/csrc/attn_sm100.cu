// attn_sm100.cu -- block-sparse (banded) attention on B200 tensor cores.
//
// Computes, per head, O = softmax(scale * Q K^T + M) V with
//   M[x, y] = 0 iff |floor(x/G) - floor(y/G)| < a, else -inf,
// the block-banded form of the spatial mask ("Sparse Video-Gen", Spatial
// Head: G = F, a = a1) and of the temporal mask after the token-major layout
// transformation ("Sparse VideoGen ...", Abstract; G = N, a = a2).  These are
// the "customized kernel implementations" the pages name without giving a
// design; the design here is B200-native.
//
// Because the band is contiguous in the key index, a query tile [q0, q1)
// only needs keys [max(0, (g(q0)-a+1) G), min(L, (g(q1-1)+a) G)).  The kernel
// derives that range from (G, a) on the fly -- no mask tensor, no block list
// in memory -- and masks elementwise only in tiles a row's band does not
// fully cover.
//
// One CTA = 256 query rows = two 128-row Q tiles sharing every K/V tile, 10
// warps:
//   warp 8      TMA producer: Q tiles once, then K_k / V_k into a ring of
//               128-key slots (128-byte swizzle, OOB rows zero-filled);
//   warp 9      one thread issues tcgen05.mma: S_i = Q_i K^T into TMEM, and
//               O_i += P_i V with P_i read straight from TMEM;
//   warps 0-3   softmax of Q tile 0, warps 4-7 softmax of Q tile 1: one thread
//               per query row reads its S row from TMEM, applies the band
//               mask on edge tiles, keeps the running max / sum, writes P as
//               bf16 back into the S columns, and rescales its O row in TMEM
//               only when the max grew by more than 2^8 (lazy rescaling).
// The MMA order S_0, S_1, then per key tile {P_0 V, S_0 <- next}, {P_1 V,
// S_1 <- next} lets the tensor core work on one Q tile while the other's
// softmax runs.  (Two issuing threads, one per tile, measured slower: the
// finely interleaved MMAs of two accumulators ran below this order's rate.)
// TMEM: S_0 [0,128) S_1 [128,256) O_0 [256,256+D) O_1 [256+D,256+2D).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"

namespace svg {

namespace {

constexpr int kMaxFrameGroups = 24;

struct AttnParams {
  CUtensorMap tm_q, tm_k, tm_v;     // frame-major, laid out as st_in
  CUtensorMap tm_qp, tm_kp, tm_vp;  // token-major, laid out as st_p
  // Fused layout transformation: 4D views (d, frame, position, head) of the
  // frame-major q/k/v whose box is s frames x 128/s positions (s = 2^e, map
  // index e): one box is a 128-row tile already in token-major order.
  CUtensorMap tm_fq[8], tm_fk[8], tm_fv[8];
  __nv_bfloat16* o;   // laid out as st_o
  __nv_bfloat16* op;  // laid out as st_p
  HeadStrides st_in, st_p, st_o;
  const int8_t* label;  // spatial (0) / temporal (1) per head, or nullptr
  const int8_t* modes;  // mixed-pattern mode per head (SVG_MODE_*), or nullptr
  int BH, L, n_ctiles;
  int G0, a0, G1, a1;
  int win, md_a, stripe, N;  // mixed modes: window half-width, multi-diagonal band, stripe length
  float sl2;      // scale * log2(e)
  float lazy_th;  // rescale threshold in raw score units (8 / sl2)
  int* status;
  uint64_t wait_ns;
  int withhold_loads;  // self-test only: the producer issues nothing
  int fused;           // token-major heads load through tm_f* and write O rows to frame-major positions
  int F;               // tokens per frame (fused only)
  // Frames split into groups of power-of-two size (largest first):
  // group g = frames [gfirst[g], gfirst[g] + 2^glog[g]); a CTA of a
  // token-major head takes 2 Q tiles of one group (2 * 128 / 2^glog[g]
  // positions).  CTAs are ordered by position: block b of bpos positions
  // has cpb CTAs, gcta[g] of them for group g (in group order), so CTAs that
  // run together share their key positions in L2.
  int ng, bpos, cpb;
  int glog[kMaxFrameGroups], gfirst[kMaxFrameGroups], gcta[kMaxFrameGroups];
  // SVG2 cluster-pair mode: see BandAttnArgs
  int s2, s2_Cq, s2_Ck, s2_W;
  const int32_t* s2_cid;
  const int32_t* s2_perm;
  const int32_t* s2_koff;
  const uint32_t* s2_sel;
};

// SVG2 key tiles: 128-row tiles over the runs of consecutive kept key
// clusters (empty clusters do not break a run; kept clusters are contiguous
// in the permuted keys).  `u` is the CTA's union of kept key clusters.
struct S2Run {
  int t, end, next;  // current tile row, end of the run, first cluster after it
};

__device__ __forceinline__ bool s2_bit(const uint32_t* u, int c) { return (u[c >> 5] >> (c & 31)) & 1u; }

// The first run at or after cluster `from`; end == -1 when there is none.
__device__ __forceinline__ S2Run s2_run(const uint32_t* u, const int32_t* koff, int Ck, int from) {
  int c = from;
  while (c < Ck && !(s2_bit(u, c) && koff[c + 1] > koff[c])) ++c;
  if (c == Ck) return S2Run{0, -1, Ck};
  int e = c + 1;
  while (e < Ck && (s2_bit(u, e) || koff[e + 1] == koff[e])) ++e;
  return S2Run{koff[c], koff[e], e};
}

__device__ __forceinline__ void s2_next(S2Run& r, const uint32_t* u, const int32_t* koff, int Ck) {
  r.t += 128;
  if (r.t >= r.end) r = s2_run(u, koff, Ck, r.next);
}

// 128-bit keep mask of one row for the tile [r.t, r.t + 128) of run r: the
// keys of the clusters the row's query cluster keeps (`row`, one bit per key
// cluster), cut at the end of the run (a run's last tile can reach into the
// next run, whose keys its own tiles count).  `kc` is the first key cluster
// that can overlap the tile; it only moves forward.
__device__ __forceinline__ void s2_tile_mask(const S2Run& r, const int32_t* koff, const uint32_t* row, int Ck,
                                             int& kc, uint32_t (&km)[4]) {
  const int t0 = r.t, lim = min(t0 + 128, r.end);
  km[0] = km[1] = km[2] = km[3] = 0u;
  while (kc < Ck - 1 && koff[kc + 1] <= t0) ++kc;
  for (int c = kc; c < Ck && koff[c] < lim; ++c) {
    if (!((row[c >> 5] >> (c & 31)) & 1u)) continue;
    const int a0 = max(koff[c], t0) - t0, a1 = min(koff[c + 1], lim) - t0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int lo = max(a0, 32 * w), hi = min(a1, 32 * w + 32);
      if (lo < hi) {
        const uint32_t hi_m = (hi - 32 * w == 32) ? 0xffffffffu : ((1u << (hi - 32 * w)) - 1u);
        km[w] |= hi_m & ~((1u << (lo - 32 * w)) - 1u);
      }
    }
  }
}

template <int D>
struct Cfg {
  static constexpr int BQ = 128;          // rows per Q tile (MMA M)
  static constexpr int BK = 128;          // keys per K/V tile
  static constexpr int HALVES = D / 64;   // 128-byte swizzle rows hold 64 bf16
  static constexpr int HALF_BYTES = 128 * 128;  // 128 rows x 128 bytes
  static constexpr int TILE_BYTES = BK * D * 2;
  static constexpr int NS = (D == 128) ? 5 : 8;  // K/V ring slots (fills shared memory)
  // d = 64: the row sums come from the tensor cores.  The P V product runs
  // with N = d + 16, its B operand V extended by a 16-column block of ones,
  // so O_i's last 16 columns accumulate sum_y P_i[x, y], the very bf16 weights
  // the product sees, in fp32.  TMEM: 2 x 128 S + 2 x 80 O columns; P is
  // written over S.
#ifndef SVG_ROWSUM_MMA
#define SVG_ROWSUM_MMA 1
#endif
  static constexpr bool ROWSUM_MMA = (D == 64) && SVG_ROWSUM_MMA;
  static constexpr int ON = D + (ROWSUM_MMA ? 16 : 0);  // O columns (+ the row-sum block)
  static constexpr int SMEM_Q = 2 * TILE_BYTES;
  static constexpr int SMEM_ONES = SMEM_Q + NS * TILE_BYTES;  // 128 rows x 64 bf16 ones (row-sum operand)
  static constexpr int SMEM_BAR = SMEM_ONES + (ROWSUM_MMA ? HALF_BYTES : 0);
  static constexpr int SMEM_BYTES = SMEM_BAR + 512 + 1024;  // barriers + alignment slack
  // 10 warps: softmax 0-3 and 4-7, TMA producer 8, MMA issuer 9.  (A 12-warp
  // layout with a setmaxnreg register split measured about 4 % slower.)
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  // d = 64 leaves TMEM room for P outside S: P_i gets its own 64 columns,
  // so S_i is free as soon as the softmax has read it and the next S_i is
  // computed while the softmax works (separate-P pipeline).  At d = 128 the
  // two O accumulators fill the rest, and P is written over S.
  static constexpr bool SEP_P = (D == 64) && !ROWSUM_MMA;
  static constexpr uint32_t col_s(int i) { return 128u * i; }
  static constexpr uint32_t col_p(int i) { return SEP_P ? 256u + 64u * i : 128u * i; }
  // O_i starts on a 32-column boundary (the epilogue loads 32 columns at a time)
  static constexpr uint32_t col_o(int i) { return SEP_P ? 384u + 64u * i : 256u + ((ON + 31) / 32 * 32) * i; }
};
// Tensor-memory and shared-memory layouts fit their allocations.
static_assert(Cfg<64>::col_s(1) + 128 <= Cfg<64>::TMEM_COLS && Cfg<64>::col_p(1) + 64 <= Cfg<64>::TMEM_COLS &&
                  Cfg<64>::col_o(1) + Cfg<64>::ON <= Cfg<64>::TMEM_COLS &&
                  (!Cfg<64>::SEP_P || (Cfg<64>::col_s(1) + 128 <= Cfg<64>::col_p(0) &&
                                       Cfg<64>::col_p(1) + 64 <= Cfg<64>::col_o(0))) &&
                  Cfg<64>::col_s(1) + 128 <= Cfg<64>::col_o(0),
              "d = 64 TMEM layout");
static_assert(Cfg<128>::col_s(1) + 128 <= Cfg<128>::col_o(0) && Cfg<128>::col_o(1) + 128 <= Cfg<128>::TMEM_COLS,
              "d = 128 TMEM layout");
static_assert(Cfg<64>::SMEM_BYTES <= 232448 && Cfg<128>::SMEM_BYTES <= 232448, "shared memory per CTA");

// Pairs (of 8) per softmax row chunk whose exponentials use the FMA-pipe
// polynomial instead of the MUFU ex2 unit.  A d = 64 tile has half the MMA
// work of a d = 128 tile for the same exponentials; its best share is lower.
template <int D>
constexpr int exp_poly_pairs() {
  return D == 64 ? 2 : 3;
}

// P_i is handed to the MMA issuer in this many column chunks: the first
// P V products run while the softmax still computes the later keys.
#ifndef SVG_P_CHUNKS
#define SVG_P_CHUNKS 2
#endif
constexpr int kPChunks = SVG_P_CHUNKS;
static_assert(kPChunks == 1 || kPChunks == 2 || kPChunks == 4, "P chunks: 1, 2 or 4");

__device__ __forceinline__ void record_timeout(const AttnParams& p, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
}

// The keys one head keeps for query row x form one interval [lo, hi):
//   GROUP  (G, a): |floor(x/G) - floor(y/G)| < a  -> [(g-a+1)G, (g+a)G), g = floor(x/G)
//   WINDOW (W):    |x - y| <= W                     -> [x-W, x+W+1)
//   PREFIX (P):    y < P                            -> [0, P)
//   SKIP:          no key (the output row is zero)
// each clipped to [0, L).  lo and hi never decrease as x grows, so a tile of
// rows [x0, x1] needs keys [lo(x0), hi(x1)).
enum BandKind { kGroup = 0, kWindow = 1, kPrefix = 2, kSkip = 3 };
struct HeadBand {
  int kind, G, a, perm;  // perm: the head runs on the token-major copies
};

__device__ __forceinline__ void row_interval(const HeadBand& b, int x, int L, int& lo, int& hi) {
  if (b.kind == kGroup) {
    const long long g = x / b.G;
    lo = static_cast<int>(max(0LL, (g - b.a + 1) * b.G));
    hi = static_cast<int>(min(static_cast<long long>(L), (g + b.a) * b.G));
  } else if (b.kind == kWindow) {
    lo = max(0, x - b.G);
    hi = min(L, x + b.G + 1);
  } else if (b.kind == kPrefix) {
    lo = 0;
    hi = min(L, b.G);
  } else {
    lo = 0;
    hi = 0;
  }
}

__device__ __forceinline__ HeadBand head_band(const AttnParams& p, int bh) {
  if (p.modes != nullptr) {
    switch (p.modes[bh]) {
      case SVG_MODE_FULL: return HeadBand{kGroup, p.L, 1, 0};
      case SVG_MODE_DIAGONAL: return HeadBand{kWindow, p.win, 0, 0};
      case SVG_MODE_MULTIDIAG: return HeadBand{kGroup, p.N, p.md_a, 1};
      case SVG_MODE_STRIPE: return HeadBand{kPrefix, p.stripe, 0, 0};
      default: return HeadBand{kSkip, 1, 0, 0};
    }
  }
  // Only SVG_TEMPORAL selects the token-major band; any other value (the -1
  // a failed profiling call writes included) runs the spatial band on the
  // frame-major tensors, as the permute and unpermute kernels move only
  // SVG_TEMPORAL heads.
  const bool temporal = p.label != nullptr && p.label[bh] == SVG_TEMPORAL;
  return temporal ? HeadBand{kGroup, p.G1, p.a1, 1} : HeadBand{kGroup, p.G0, p.a0, 0};
}

// Warp-uniform bounded wait.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, limit);
  return __all_sync(0xffffffffu, ok);
}

// S2: the SVG2 cluster-pair mode (its own instantiation, so the other modes
// keep their register allocation).
template <int D, bool S2>
__global__ void __launch_bounds__(320, 1) attn_sm100_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::SMEM_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bars + 1 + C::NS;
  uint64_t* bar_s = bars + 1 + 2 * C::NS;  // [2] S_i ready
  uint64_t* bar_p = bar_s + 2;             // [2][kPChunks] chunk of P_i written (128 arrivals)
  uint64_t* bar_o = bar_p + 2 * kPChunks;  // [2] P_i V done
  uint64_t* bar_sfree = bar_o + 2;         // [2] separate-P pipeline: S_i read by the softmax (128 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_sfree + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* s2u = reinterpret_cast<uint32_t*>(tmem_slot + 2);  // [32] SVG2: union of kept key clusters

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) & SVG_DEV_TIMEOUT) ? 1 : 0;
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s[i], 1);
      for (int j = 0; j < kPChunks; ++j) mbar_init(&bar_p[i * kPChunks + j], 128);
      mbar_init(&bar_o[i], 1);
      mbar_init(&bar_sfree[i], 128);
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (C::ROWSUM_MMA) {
    // the ones block of the row-sum product (bf16 1.0 = 0x3F80), made visible
    // to the tensor cores' (async-proxy) reads
    uint4* ones = reinterpret_cast<uint4*>(smem + C::SMEM_ONES);
    for (int e = threadIdx.x; e < C::HALF_BYTES / 16; e += C::THREADS)
      ones[e] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (S2 && threadIdx.x < p.s2_W) {
    // union of the key clusters kept by the query clusters of this CTA's rows
    const int bh_ = blockIdx.x / p.n_ctiles, q0_ = (blockIdx.x % p.n_ctiles) * 256;
    uint32_t w = 0;
    if (q0_ < p.L) {
      const int32_t* cid = p.s2_cid + static_cast<size_t>(bh_) * p.L;
      const int c0 = cid[q0_], c1 = cid[min(q0_ + 255, p.L - 1)];
      for (int c = c0; c <= c1; ++c) w |= p.s2_sel[(static_cast<size_t>(bh_) * p.s2_Cq + c) * p.s2_W + threadIdx.x];
    }
    s2u[threadIdx.x] = w;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- work item: (head, 256-row query slab)
  const int ct = blockIdx.x % p.n_ctiles;
  const int bh = blockIdx.x / p.n_ctiles;
  const HeadBand band = head_band(p, bh);
  const int lab = band.perm;
  const bool fz = lab && p.fused && !S2;  // token-major head, layout transformation fused into the loads
  const int L = p.L;
  bool idle = false;  // no query rows for this CTA
  int q0 = 0, kt0 = 0, nk = 0;
  // fused: Q tile group, its first position, and the key position range
  int gq = 0, pq0 = 0, kp_lo = 0, kp_hi = 0;
  const int32_t* s2_koff = S2 ? p.s2_koff + static_cast<size_t>(bh) * (p.s2_Ck + 1) : nullptr;
  if (S2) {
    if (ct * 256 >= L) {
      idle = true;
    } else {
      q0 = ct * 256;
      for (S2Run r = s2_run(s2u, s2_koff, p.s2_Ck, 0); r.end >= 0; r = s2_run(s2u, s2_koff, p.s2_Ck, r.next))
        nk += (r.end - r.t + C::BK - 1) / C::BK;
    }
  } else if (fz) {
    const int blk = ct / p.cpb;
    int rem = ct - blk * p.cpb;
    while (gq < p.ng && rem >= p.gcta[gq]) rem -= p.gcta[gq++];
    const int shq = 7 - p.glog[gq < p.ng ? gq : 0];  // log2 of positions per Q tile
    pq0 = blk * p.bpos + (rem << (shq + 1));
    if (gq == p.ng || pq0 >= p.F) {
      idle = true;
    } else {
      const int pq_hi = min(p.F - 1, pq0 + (2 << shq) - 1);
      kp_lo = max(0, pq0 - band.a + 1);
      kp_hi = min(p.F - 1, pq_hi + band.a - 1);
      for (int g = 0; g < p.ng; ++g) {
        const int sh = 7 - p.glog[g];
        nk += (kp_hi >> sh) - (kp_lo >> sh) + 1;
      }
    }
  } else if (ct * 256 >= L) {
    idle = true;
  } else {
    q0 = ct * 256;
    const int q_last = min(q0 + 255, L - 1);
    int lo_cta, hi_cta, lo_unused, hi_unused;
    row_interval(band, q0, L, lo_cta, hi_unused);
    row_interval(band, q_last, L, lo_unused, hi_cta);
    kt0 = lo_cta / C::BK;
    nk = (hi_cta > lo_cta) ? (hi_cta + C::BK - 1) / C::BK - kt0 : 0;  // 0: skipped head
  }
  const bool run = (*abort_flag == 0);
  const int th_in = p.st_in.tma_h(bh), tb_in = p.st_in.tma_b(bh);  // TMA (head, batch) of q, k, v

  if (warp >= 8) {
    if (run && nk > 0 && warp == 8 && lane == 0 && !p.withhold_loads && fz) {
      // ------------------------------------------------ TMA producer, fused layout transformation
      // Key tiles go group by group; within group g, tile t holds positions
      // [t P, (t+1) P) (P = 128 / 2^glog[g]) of the group's frames, one 4D box
      // per 64-column half.  Positions past F read zeros.
      tma_prefetch_desc(&p.tm_fq[p.glog[gq]]);
      mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
      const int shq = 7 - p.glog[gq];
      in_range(pq0, p.F, p.status);
      in_range(p.gfirst[gq] + (1 << p.glog[gq]) - 1, p.N, p.status);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_5d(sQ + i * C::TILE_BYTES + h * C::HALF_BYTES, &p.tm_fq[p.glog[gq]], bar_q, h * 64,
                      p.gfirst[gq], pq0 + (i << shq), th_in, tb_in);
      int g = 0, sh = 7 - p.glog[0], t = kp_lo >> sh, t_end = kp_hi >> sh;
      for (int n = 0; n < 2 * nk; ++n) {
        const int slot = n % C::NS;
        const uint32_t ph = (n / C::NS) & 1;
        if (!mbar_wait(&bar_empty[slot], ph ^ 1, p.wait_ns)) {
          record_timeout(p, abort_flag);
          break;
        }
        const CUtensorMap* tm = (n & 1) ? &p.tm_fv[p.glog[g]] : &p.tm_fk[p.glog[g]];
        in_range(t << sh, p.F, p.status);  // key tiles start inside the head (checked build: reported)
        in_range(p.gfirst[g] + (1 << p.glog[g]) - 1, p.N, p.status);
        mbar_arrive_expect_tx(&bar_full[slot], C::TILE_BYTES);
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_5d(sRing + slot * C::TILE_BYTES + h * C::HALF_BYTES, tm, &bar_full[slot], h * 64, p.gfirst[g],
                      t << sh, th_in, tb_in);
        if ((n & 1) && ++t > t_end && ++g < p.ng) {  // next key tile after its V
          sh = 7 - p.glog[g];
          t = kp_lo >> sh;
          t_end = kp_hi >> sh;
        }
      }
    } else if (run && nk > 0 && warp == 8 && lane == 0 && !p.withhold_loads && S2) {
      // ------------------------------------------------ TMA producer, SVG2 cluster runs
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_4d(sQ + i * C::TILE_BYTES + h * C::HALF_BYTES, &p.tm_q, bar_q, h * 64, q0 + i * C::BQ, th_in,
                      tb_in);
      S2Run kr = s2_run(s2u, s2_koff, p.s2_Ck, 0);
      for (int n = 0; n < 2 * nk; ++n) {
        const int slot = n % C::NS;
        const uint32_t ph = (n / C::NS) & 1;
        if (!mbar_wait(&bar_empty[slot], ph ^ 1, p.wait_ns)) {
          record_timeout(p, abort_flag);
          break;
        }
        const CUtensorMap* tm = (n & 1) ? &p.tm_v : &p.tm_k;
        in_range(kr.t, L, p.status);
        mbar_arrive_expect_tx(&bar_full[slot], C::TILE_BYTES);
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_4d(sRing + slot * C::TILE_BYTES + h * C::HALF_BYTES, tm, &bar_full[slot], h * 64, kr.t, th_in,
                      tb_in);
        if (n & 1) s2_next(kr, s2u, s2_koff, p.s2_Ck);
      }
    } else if (run && nk > 0 && warp == 8 && lane == 0 && !p.withhold_loads) {
      // ------------------------------------------------ TMA producer
      {
      const CUtensorMap* tq = lab ? &p.tm_qp : &p.tm_q;
      const CUtensorMap* tk = lab ? &p.tm_kp : &p.tm_k;
      const CUtensorMap* tv = lab ? &p.tm_vp : &p.tm_v;
      const int th = lab ? p.st_p.tma_h(bh) : th_in, tb = lab ? p.st_p.tma_b(bh) : tb_in;
      tma_prefetch_desc(tq);
      tma_prefetch_desc(tk);
      tma_prefetch_desc(tv);
      in_range(q0, L, p.status);
      mbar_arrive_expect_tx(bar_q, 2 * C::TILE_BYTES);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_4d(sQ + i * C::TILE_BYTES + h * C::HALF_BYTES, tq, bar_q, h * 64, q0 + i * C::BQ, th, tb);
      for (int n = 0; n < 2 * nk; ++n) {
        const int slot = n % C::NS;
        const uint32_t ph = (n / C::NS) & 1;
        if (!mbar_wait(&bar_empty[slot], ph ^ 1, p.wait_ns)) {
          record_timeout(p, abort_flag);
          break;
        }
        const CUtensorMap* tm = (n & 1) ? tv : tk;
        const int row = (kt0 + (n >> 1)) * C::BK;
        in_range(row, L, p.status);
        mbar_arrive_expect_tx(&bar_full[slot], C::TILE_BYTES);
#pragma unroll
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_4d(sRing + slot * C::TILE_BYTES + h * C::HALF_BYTES, tm, &bar_full[slot], h * 64, row, th, tb);
      }
    }
    } else if (run && nk > 0 && warp == 9) {
      // ------------------------------------------------ MMA issuer
      // The whole warp runs this loop (waits, descriptor arithmetic) in
      // lockstep, and one elected lane issues each tcgen05 instruction: the
      // operands stay warp-uniform, which keeps the per-MMA issue cost low
      // while the softmax warps on the same sub-partition keep it busy.
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::ON, 0, 1);
      const uint32_t ring_base = smem_u32(sRing);
      // Descriptors are built once; offsets go into the start-address field
      // (address >> 4 in the low bits; every operand lies below 256 KB).
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = smem_desc_sw128(ring_base, 16, 1024);
      const uint64_t dv = smem_desc_sw128(ring_base, C::HALF_BYTES, 1024);
      auto issue_qk = [&](int i, int slot) {
        const uint64_t a = dq + static_cast<uint64_t>((i * C::TILE_BYTES) >> 4);
        const uint64_t b = dk + static_cast<uint64_t>((slot * C::TILE_BYTES) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::HALF_BYTES + (kk & 3) * 32) >> 4);
          umma_ss_warp(tmem + C::col_s(i), a + off, b + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit_warp(&bar_s[i]);
      };
      // The P V products of one chunk of P_i (keys [j, j+1) * BK / kPChunks).
      const uint32_t ones_addr = smem_u32(smem + C::SMEM_ONES);
      auto issue_pv_chunk = [&](int i, int slot, bool acc, int j) {
        // row-sum form: the ones block is V's second 64-column block, one
        // leading-dimension offset past the slot (a per-slot offset)
        const uint32_t vslot = ring_base + slot * C::TILE_BYTES;
        const uint64_t b = C::ROWSUM_MMA ? smem_desc_sw128(vslot, ones_addr - vslot, 1024)
                                         : dv + static_cast<uint64_t>((slot * C::TILE_BYTES) >> 4);
        constexpr int KK = C::BK / 16 / kPChunks;
#pragma unroll
        for (int u = 0; u < KK; ++u) {
          const int kk = j * KK + u;
          umma_ts_warp(tmem + C::col_o(i), tmem + C::col_p(i) + kk * 8,
                       b + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = warp_wait(bar_q, 0, p.wait_ns) && warp_wait(&bar_full[0], 0, p.wait_ns);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
        umma_commit_warp(&bar_empty[0]);
      }
      for (int k = 0; ok && C::SEP_P && k < nk; ++k) {
        // separate-P pipeline: S_i <- K_{k+1} as soon as the softmax has read
        // S_i (it writes P_i to its own columns), then O_i += P_i V_k once P_i
        // is written.  The next scores are ready before the softmax needs them.
        const int nV = 2 * k + 1, nK = 2 * k + 2;
        const int slotV = nV % C::NS, slotK = nK % C::NS;
        if (k + 1 < nk) {
          ok = warp_wait(&bar_full[slotK], (nK / C::NS) & 1, p.wait_ns);
          for (int i = 0; ok && i < 2; ++i) {
            ok = warp_wait(&bar_sfree[i], k & 1, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_qk(i, slotK);
          }
          if (!ok) break;
          umma_commit_warp(&bar_empty[slotK]);
        }
        ok = warp_wait(&bar_full[slotV], (nV / C::NS) & 1, p.wait_ns);
        for (int i = 0; ok && i < 2; ++i) {
#pragma unroll
          for (int j = 0; j < kPChunks; ++j) {
            ok = warp_wait(&bar_p[i * kPChunks + j], k & 1, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_pv_chunk(i, slotV, k > 0, j);
          }
          if (!ok) break;
          umma_commit_warp(&bar_o[i]);  // O_i holds P_i V_k and P_i may be overwritten
        }
        if (!ok) break;
        umma_commit_warp(&bar_empty[slotV]);
      }
      for (int k = 0; ok && !C::SEP_P && k < nk; ++k) {
        const int nV = 2 * k + 1, nK = 2 * k + 2;
        const int slotV = nV % C::NS, slotK = nK % C::NS;
        const bool has_next = k + 1 < nk;
        ok = warp_wait(&bar_full[slotV], (nV / C::NS) & 1, p.wait_ns);
        for (int i = 0; ok && i < 2; ++i) {
#pragma unroll
          for (int j = 0; j < kPChunks; ++j) {
            ok = warp_wait(&bar_p[i * kPChunks + j], k & 1, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            issue_pv_chunk(i, slotV, k > 0, j);
          }
          if (!ok) break;
          umma_commit_warp(&bar_o[i]);
          // V_k is free once both tiles' P V products have read it.
          if (i == 1) umma_commit_warp(&bar_empty[slotV]);
          if (has_next) {
            if (i == 0) {
              ok = warp_wait(&bar_full[slotK], (nK / C::NS) & 1, p.wait_ns);
              if (!ok) break;
              tc_fence_after();
            }
            issue_qk(i, slotK);
          }
        }
        if (!ok) break;
        if (has_next) umma_commit_warp(&bar_empty[slotK]);
      }
      if (!ok && lane == 0) record_timeout(p, abort_flag);
    }
  } else {
    if (run) {
    // ------------------------------------------------ softmax / epilogue
    const int i = warp >> 2;
    const int quad = warp & 3;
    const int r = q0 + i * C::BQ + quad * 32 + lane;  // query row in the head's layout (unfused)
    // fused: the row's position and frame (rows of a tile: position-major,
    // the group's frames inside), and its frame-major row x = frame F + pos
    int pos_q = 0, x_q = r;
    if (fz) {
      const int rt = quad * 32 + lane;
      const int lg = p.glog[gq];
      pos_q = pq0 + (i << (7 - lg)) + (rt >> lg);
      x_q = (p.gfirst[gq] + (rt & ((1 << lg) - 1))) * p.F + pos_q;
    }
    const bool row_ok = !idle && (fz ? pos_q < p.F : r < L);
    int lo_r = 0, hi_r = 0;
    if (row_ok && !fz && !S2) row_interval(band, r, L, lo_r, hi_r);
    // SVG2: the row's kept key clusters, the key run iterator, and the first
    // key cluster that can overlap the current tile
    const uint32_t* s2_row = nullptr;
    S2Run s2r{0, -1, 0};
    int s2_kc = 0;
    uint32_t s2_km[4] = {0u, 0u, 0u, 0u};  // keep mask of the next tile, built ahead of its scores
    if (S2) {
      int cq = row_ok ? p.s2_cid[static_cast<size_t>(bh) * L + r] : 0;
      if (!in_range(cq, p.s2_Cq, p.status)) cq = 0;
      s2_row = p.s2_sel + (static_cast<size_t>(bh) * p.s2_Cq + cq) * p.s2_W;
      if (!idle) s2r = s2_run(s2u, s2_koff, p.s2_Ck, 0);
      if (S2 && row_ok) x_q = p.s2_perm[static_cast<size_t>(bh) * L + r];
      if (S2 && row_ok && !in_range(x_q, L, p.status)) x_q = 0;
      if (nk > 0) s2_tile_mask(s2r, s2_koff, s2_row, p.s2_Ck, s2_kc, s2_km);
    }
    int kg = 0, ksh = 7 - p.glog[0], kt = kp_lo >> ksh, kt_end = kp_hi >> ksh;  // fused key-tile iterator
    const uint32_t lane_bits = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + lane_bits + C::col_s(i);
    const uint32_t tP = tmem + lane_bits + C::col_p(i);
    const uint32_t tO = tmem + lane_bits + C::col_o(i);
    const float sl2 = p.sl2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int k = 0; k < nk; ++k) {
      if (!warp_wait(&bar_s[i], k & 1, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence32(sr[c]);
      if (C::SEP_P) {  // S_i has been read: the next scores may overwrite it
        tc_fence_before();
        mbar_arrive(&bar_sfree[i]);
      }
      float s[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(sr[c][e]);

      // keys of this tile the row keeps: columns [lo_c, hi_c)
      int lo_c, hi_c;
      if (S2) {
        // the keep mask of this tile was built while its scores were computed
        if ((s2_km[0] & s2_km[1] & s2_km[2] & s2_km[3]) != 0xffffffffu) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (!((s2_km[c >> 5] >> (c & 31)) & 1u)) s[c] = -INFINITY;
        }
        lo_c = 0;
        hi_c = C::BK;
      } else if (fz) {
        // key column c holds position (kt << ksh) + (c >> lg) of the group
        const int lg = 7 - ksh, p0 = kt << ksh;
        lo_c = (pos_q - band.a + 1 - p0) * (1 << lg);
        hi_c = (min(pos_q + band.a, p.F) - p0) * (1 << lg);
        if (++kt > kt_end && ++kg < p.ng) {
          ksh = 7 - p.glog[kg];
          kt = kp_lo >> ksh;
          kt_end = kp_hi >> ksh;
        }
      } else {
        const int kbase = (kt0 + k) * C::BK;
        lo_c = lo_r - kbase;
        hi_c = hi_r - kbase;
      }
      if (lo_c > 0 || hi_c < C::BK) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c < lo_c || c >= hi_c) s[c] = -INFINITY;
      }
      float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]), mx2 = fmaxf(s[4], s[5]), mx3 = fmaxf(s[6], s[7]);
#pragma unroll
      for (int c = 8; c < 128; c += 8) {
        mx0 = fmax3f(mx0, s[c], s[c + 1]);
        mx1 = fmax3f(mx1, s[c + 2], s[c + 3]);
        mx2 = fmax3f(mx2, s[c + 4], s[c + 5]);
        mx3 = fmax3f(mx3, s[c + 6], s[c + 7]);
      }
      const float m_new = fmax3f(m_used, fmax3f(mx0, mx1, mx2), mx3);
      float alpha = 1.f;
      bool resc = false;
      if (m_new > m_used + p.lazy_th) {  // false while both are -inf
        alpha = ex2_approx((m_used - m_new) * sl2);  // 0 when m_used is -inf
        m_used = m_new;
        resc = true;
      }
      l *= alpha;
      // O_i rescale (separate-P pipeline: just before P_i is overwritten, below)
      auto rescale_o = [&]() {
#pragma unroll 1
        for (int c = 0; c < C::ON / 16; ++c) {  // with the row-sum columns, if any
          uint32_t ov[16];
          tmem_ld16(tO + c * 16, ov);
          tmem_wait_ld();
          reg_fence16(ov);
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st16(tO + c * 16, ov);
        }
      };
      const bool any_resc = k > 0 && __any_sync(0xffffffffu, resc);
      if (!C::SEP_P && any_resc) {
        // O_i holds P_i(k-1) V (its product completed before S_i(k) did);
        // rescale it before any P_i(k) V product is issued.
        if (!warp_wait(&bar_o[i], (k - 1) & 1, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 16 columns at a time: the 128 scores stay live in registers here
        rescale_o();
      }
      const float nb = (m_used == -INFINITY) ? 0.f : -m_used * sl2;
      const float2 sl2x2 = make_float2(sl2, sl2), nb2 = make_float2(nb, nb);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      constexpr int PPC = 64 / kPChunks;  // key pairs (P columns) per chunk
#pragma unroll
      for (int j = 0; j < kPChunks; ++j) {
        uint32_t pk[PPC];
#pragma unroll
        for (int cc = 0; cc < PPC; ++cc) {
          const int c = j * PPC + cc;
          const float2 x = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sl2x2, nb2);
          float2 pr;
          if ((c & 7) < exp_poly_pairs<D>()) {  // a fixed share of the pairs on the FMA pipe
            pr = exp2_poly2(x);
          } else {
            pr.x = ex2_approx(x.x);
            pr.y = ex2_approx(x.y);
          }
          const uint32_t pp = pack_bf16x2(pr.x, pr.y);
          // The row sum uses the same bf16-rounded weights the P V product
          // sees, so each output row is an exact convex combination of V rows
          // (with ROWSUM_MMA the tensor cores add them up in O's last columns).
          if (!C::ROWSUM_MMA) {
            if (c & 1) add_bf16x2_f32(acc1, pp);
            else add_bf16x2_f32(acc0, pp);
          }
          pk[cc] = pp;
        }
        if (C::SEP_P && j == 0 && k > 0) {
          // P_i(k-1) V done: P_i may be overwritten and O_i holds it (the
          // products of tile k-2 finished before S_i(k) was computed, those
          // of tile k wait for this P, so the parity identifies the phase)
          if (!warp_wait(&bar_o[i], (k - 1) & 1, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (any_resc) rescale_o();
        }
        __syncwarp();
#pragma unroll
        for (int h = 0; h < PPC / 16; ++h) tmem_st16(tP + j * PPC + h * 16, pk + h * 16);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_p[i * kPChunks + j]);
      }
      if (!ok) break;
      l += (acc0.x + acc1.x) + (acc0.y + acc1.y);
      if (S2 && k + 1 < nk) {
        // the next tile's keep mask, while the tensor cores compute its scores
        s2_next(s2r, s2u, s2_koff, p.s2_Ck);
        s2_tile_mask(s2r, s2_koff, s2_row, p.s2_Ck, s2_kc, s2_km);
      }
    }
    if (idle) {
      // no query rows here
    } else if (nk == 0) {
      // skipped head: its output rows are zero
      if (row_ok && in_range(x_q, L, p.status) && in_range(bh, p.BH, p.status)) {
        const bool to_op = lab && !p.fused && !S2;
        const HeadStrides& so = to_op ? p.st_p : p.st_o;
        uint4* dst = reinterpret_cast<uint4*>((to_op ? p.op : p.o) + so.head(bh) + x_q * so.sl);
#pragma unroll
        for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
      }
    } else if (ok && warp_wait(&bar_o[i], (nk - 1) & 1, p.wait_ns)) {
      tc_fence_after();
      if (C::ROWSUM_MMA) {  // the row sum is column D of O_i
        uint32_t lv[16];
        __syncwarp();
        tmem_ld16(tO + D, lv);
        tmem_wait_ld();
        reg_fence16(lv);
        l = __uint_as_float(lv[0]);
      }
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      // output row: token-major heads write to op, or, fused, straight to
      // the frame-major position of their row in o
      const bool store_ok = row_ok && in_range(x_q, L, p.status) && in_range(bh, p.BH, p.status);
      const int orow = store_ok ? x_q : 0;
      const bool to_op = lab && !p.fused && !S2;
      const HeadStrides& so = to_op ? p.st_p : p.st_o;
      __nv_bfloat16* out = (to_op ? p.op : p.o) + so.head(store_ok ? bh : 0) + orow * so.sl;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        __syncwarp();
        tmem_ld32(tO + c * 32, ov);
        tmem_wait_ld();
        reg_fence32(ov);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(ov[2 * e]) * inv_l, __uint_as_float(ov[2 * e + 1]) * inv_l);
        if (store_ok) {
          uint4* dst = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    } else {
      record_timeout(p, abort_flag);
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side

template <int D>
svg_status launch_d(const BandAttnArgs& a, cudaStream_t stream) {
  using C = Cfg<D>;
  AttnParams p;
  memset(&p, 0, sizeof(p));
  const int BH = a.B * a.H;
  svg_status st;
  const bool perm = (a.label != nullptr || a.modes != nullptr) && !a.fused;
  // q, k, v: the caller's, or in the SVG2 mode the cluster-permuted copies;
  // qp..op: the token-major copies, standing in for q..o when unused
  p.st_in = a.s2 ? a.hsp : a.hs;
  p.st_p = perm ? a.hsp : p.st_in;
  p.st_o = a.hs;
  if ((st = make_tile_map_bf16(&p.tm_q, a.q, p.st_in, a.L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_k, a.k, p.st_in, a.L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_v, a.v, p.st_in, a.L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_qp, perm ? a.qp : a.q, p.st_p, a.L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_kp, perm ? a.kp : a.k, p.st_p, a.L, D)) != SVG_OK) return st;
  if ((st = make_tile_map_bf16(&p.tm_vp, perm ? a.vp : a.v, p.st_p, a.L, D)) != SVG_OK) return st;
  p.fused = a.fused;
  p.F = a.N > 0 ? a.L / a.N : 0;
  p.s2 = a.s2;
  if (a.s2) {
    if (a.s2_Ck < 1 || a.s2_Ck > 1024 || a.s2_Cq < 1) return fail(SVG_ERR_INVALID_ARG, "cluster counts");
    p.s2_Cq = a.s2_Cq;
    p.s2_Ck = a.s2_Ck;
    p.s2_W = (a.s2_Ck + 31) / 32;
    p.s2_cid = a.s2_cid;
    p.s2_perm = a.s2_perm;
    p.s2_koff = a.s2_koff;
    p.s2_sel = a.s2_sel;
  }
  int perm_ctas = 0;
  if (a.fused) {
    if (a.N < 1 || a.L % a.N != 0) return fail(SVG_ERR_INVALID_ARG, "fused layout transformation needs N >= 1");
    p.ng = fused_frame_groups(a.N, p.glog, kMaxFrameGroups);
    if (p.ng < 0) return fail(SVG_ERR_UNSUPPORTED, "too many frames for the fused layout (N = %d)", a.N);
    for (int g = 0, first = 0; g < p.ng; ++g) {
      p.gfirst[g] = first;
      first += 1 << p.glog[g];
    }
    // position blocks: as wide as the smallest group's CTA (2 * 128 / 2^lg
    // positions); group g has bpos / (2 * 128 >> lg) CTAs per block
    p.bpos = 2 * (128 >> p.glog[p.ng - 1]);
    p.cpb = 0;
    for (int g = 0; g < p.ng; ++g) {
      p.gcta[g] = p.bpos / (2 * (128 >> p.glog[g]));
      p.cpb += p.gcta[g];
    }
    perm_ctas = (p.F + p.bpos - 1) / p.bpos * p.cpb;
    bool made[8] = {false, false, false, false, false, false, false, false};
    for (int g = 0; g < p.ng; ++g) {
      const int lg = p.glog[g];
      if (made[lg]) continue;
      made[lg] = true;
      if ((st = make_group_map_bf16(&p.tm_fq[lg], a.q, p.st_in, a.N, p.F, D, 1 << lg)) != SVG_OK) return st;
      if ((st = make_group_map_bf16(&p.tm_fk[lg], a.k, p.st_in, a.N, p.F, D, 1 << lg)) != SVG_OK) return st;
      if ((st = make_group_map_bf16(&p.tm_fv[lg], a.v, p.st_in, a.N, p.F, D, 1 << lg)) != SVG_OK) return st;
    }
  }
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.op = static_cast<__nv_bfloat16*>(perm ? a.op : a.o);
  p.label = a.label;
  p.modes = a.modes;
  p.win = a.win;
  p.md_a = a.md_a;
  p.stripe = a.stripe;
  p.N = a.N;
  p.BH = BH;
  p.L = a.L;
  p.n_ctiles = (a.L + 255) / 256;
  if (perm_ctas > p.n_ctiles) p.n_ctiles = perm_ctas;  // CTAs past a head's own count are idle
  p.G0 = a.G0;
  p.a0 = a.a0;
  p.G1 = a.G1;
  p.a1 = a.a1;
  p.sl2 = a.scale * 1.4426950408889634f;
  p.lazy_th = 8.0f / p.sl2;
  p.status = a.status;
  p.wait_ns = a.wait_ns;
  p.withhold_loads = a.withhold_loads;
  const long long grid = static_cast<long long>(BH) * p.n_ctiles;
  if (grid > 0x7fffffffLL) return fail(SVG_ERR_UNSUPPORTED, "grid too large");
  static bool attr_set[2] = {false, false};
  if (!attr_set[a.s2 ? 1 : 0]) {
    cudaError_t e = a.s2 ? cudaFuncSetAttribute(attn_sm100_kernel<D, true>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)
                         : cudaFuncSetAttribute(attn_sm100_kernel<D, false>,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute(attention smem)");
    attr_set[a.s2 ? 1 : 0] = true;
  }
  if (a.s2)
    attn_sm100_kernel<D, true><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(p);
  else
    attn_sm100_kernel<D, false><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cuda_check(cudaGetLastError(), "attention launch");
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 4D view (d, row, head, batch entry): box = 64 elements x 128 rows, 128-byte
// swizzle.  In [B, L, H, d] the row stride exceeds the head stride, so the
// strides need not increase with the dimension.
svg_status make_tile_map_bf16(CUtensorMap* map, const void* base, const HeadStrides& s, int L, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return fail(SVG_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(s.H),
                              static_cast<cuuint64_t>(s.nb)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.sl) * 2, static_cast<cuuint64_t>(s.sh) * 2,
                                 static_cast<cuuint64_t>(s.sb) * 2};
  const cuuint32_t box[4] = {64, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return SVG_OK;
}

// 5D view (d, frame, position, head, batch entry) of a frame-major tensor
// with a box of `size` frames x 128/size positions: the box's 128 rows come
// out position-major, i.e. in the token-major order of those frames.  The
// frame dimension has the larger stride, so the box walks frames fastest.
svg_status make_group_map_bf16(CUtensorMap* map, const void* base, const HeadStrides& s, int N, int F, int D,
                               int size) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return fail(SVG_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(F),
                              static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.nb)};
  const cuuint64_t strides[4] = {static_cast<cuuint64_t>(F) * s.sl * 2, static_cast<cuuint64_t>(s.sl) * 2,
                                 static_cast<cuuint64_t>(s.sh) * 2, static_cast<cuuint64_t>(s.sb) * 2};
  const cuuint32_t box[5] = {64, static_cast<cuuint32_t>(size), static_cast<cuuint32_t>(128 / size), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(SVG_ERR_CUDA, "cuTensorMapEncodeTiled (frame-group map, %d frames) failed (%d)", size,
                static_cast<int>(r));
  return SVG_OK;
}

int fused_frame_groups(int N, int* glog, int max_groups) {
  int ng = 0;
  for (int left = N; left > 0; ++ng) {
    if (ng == max_groups) return -1;
    int lg = 0;
    while (lg < 7 && (2 << lg) <= left) ++lg;
    glog[ng] = lg;
    left -= 1 << lg;
  }
  return ng;
}

void token_major_tile_counts(int N, int F, int a, long long* separate, long long* fused) {
  const long long L = static_cast<long long>(N) * F;
  long long sep = 0;
  for (long long q0 = 0; q0 < L; q0 += 256) {  // 256-row query slabs of the token-major layout
    const long long q1 = std::min(q0 + 255, L - 1);
    const long long lo = std::max(0LL, (q0 / N - a + 1) * N), hi = std::min(L, (q1 / N + a) * N);
    sep += (hi + 127) / 128 - lo / 128;
  }
  *separate = sep;
  int glog[kMaxFrameGroups];
  const int ng = fused_frame_groups(N, glog, kMaxFrameGroups);
  if (ng < 0) {
    *fused = -1;
    return;
  }
  const int bpos = 2 * (128 >> glog[ng - 1]);
  long long fz = 0;
  for (int p0 = 0; p0 < F; p0 += bpos)
    for (int g = 0; g < ng; ++g) {
      const int per = 2 * (128 >> glog[g]);  // positions per CTA of group g
      for (int pq0 = p0; pq0 < p0 + bpos && pq0 < F; pq0 += per) {
        const int pq_hi = std::min(F - 1, pq0 + per - 1);
        const int kp_lo = std::max(0, pq0 - a + 1), kp_hi = std::min(F - 1, pq_hi + a - 1);
        for (int gk = 0; gk < ng; ++gk) {
          const int sh = 7 - glog[gk];
          fz += (kp_hi >> sh) - (kp_lo >> sh) + 1;
        }
      }
    }
  *fused = fz;
}

bool fused_layout_preferred(int N, int F, int a) {
  long long sep = 0, fz = 0;
  token_major_tile_counts(N, F, a, &sep, &fz);
  return fz >= 0 && fz * 100 <= sep * 103;
}

svg_status launch_attn_sm100(const BandAttnArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 64: return launch_d<64>(a, stream);
    case 128: return launch_d<128>(a, stream);
    default: return fail(SVG_ERR_UNSUPPORTED, "bf16 attention supports d in {64, 128}, got %d", a.d);
  }
}

}  // namespace svg
