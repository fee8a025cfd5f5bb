// attn_tf32.cu -- banded attention for fp32 tensors on the tcgen05 tensor
// cores in tf32 (svg_dtype SVG_TF32).
//
// The same masks as the other attention kernels: keep (x, y) iff
// |floor(x/G) - floor(y/G)| < a ("Sparse Video-Gen", Spatial Head with G = F,
// a = a1; Temporal Head after the token-major layout transformation with
// G = N, a = a2), so a query row keeps one key interval [lo, hi).
//
// One CTA per (head, 128-row query tile), one key tile of 128 rows at a time:
//   S_k = Q K_k^T      D/8 tcgen05.mma kind::tf32 (K = 8) into TMEM
//   P = exp2(S - m)    fp32 softmax, P rounded to tf32 and written over S_k
//   O += P V_k         16 tcgen05.mma kind::tf32 with A = P from TMEM
// Two S buffers: S_{k+1} is computed while the softmax works on S_k, and
// P_k V_k follows.
// Q, K and V stay fp32 in memory; the tensor cores read their top 19 bits
// (tf32), the softmax, the row sums and the accumulators are fp32.  P is
// rounded to tf32 before both its row sum and the product, so each output row
// is an exact convex combination of the tf32 rows of V.
//
// Operands are 32-column blocks (128 rows x 128 bytes): Q and K K-major with
// the 128-byte swizzle of 16-byte chunks for S; V MN-major for P V, where
// tf32 needs the 128-byte swizzle of 32-byte chunks (TMA
// CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B, descriptor layout 1: 4-row atoms of
// 512 bytes).  Warps 0-3 own the query rows
// (two threads per row: warps w and w + 4 take keys [0, 64) and [64, 128) of
// row 32 (w & 3) + lane = TMEM lane, and exchange their maxima once per tile
// through shared memory), warp 8 issues the TMA loads of a ring of
// K and V tiles (in the order the MMAs take them: K_0, K_1, V_0, K_2, V_1,
// ...), warp 9 the MMAs.  TMEM: S / P of even tiles in columns [0, 128), of
// odd tiles in [128, 256), O in [256, 256 + D).
#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

template <int D>
struct TCfg {
  static constexpr int BLOCKS = D / 32;                  // 32-column (128-byte) blocks per row
  static constexpr int BLK_BYTES = 128 * 128;            // one block of 128 rows
  static constexpr int TILE_BYTES = BLOCKS * BLK_BYTES;  // 128 rows x D fp32
  // K / V ring slots; the shared memory also keeps a second CTA (which would
  // wait for the 512 TMEM columns) off the SM
  static constexpr int NS = (D == 128) ? 2 : (D == 64) ? 4 : 8;
  static constexpr int SMEM_BAR = TILE_BYTES * (1 + NS);
  static constexpr int SMEM_X = SMEM_BAR + 256;               // half-row maxima [2][2][128], sums [2][128]
  static constexpr int SMEM_BYTES = SMEM_X + 3072 + 1024;     // 1024-byte alignment slack
  static constexpr int THREADS = 320;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t COL_O = 256;
  static_assert(COL_O + D <= TMEM_COLS, "two S buffers and O must fit the TMEM allocation");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(2 * SMEM_BYTES > 228 * 1024, "one CTA per SM");
};

struct Tf32Params {
  CUtensorMap tm_q, tm_k, tm_v;     // frame-major (or all heads without labels), laid out as st_in
  CUtensorMap tm_qp, tm_kp, tm_vp;  // token-major copies, laid out as st_p
  float* o;                          // laid out as st_in
  float* op;                         // laid out as st_p
  HeadStrides st_in, st_p;
  const int8_t* label;  // SVG_TEMPORAL heads use band 1 on the token-major copies; nullptr: band 0 everywhere
  int BH, L, n_qt;
  int G0, a0, G1, a1;
  float sl2;  // scale * log2(e)
  int* status;
  uint64_t wait_ns;
};

__device__ __forceinline__ void ss_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void ts_tf32(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::tf32, fp32 accumulator: D format (bits 4-5)
// 1 = f32, A and B formats (bits 7-9, 10-12) 2 = tf32, A / B major (15, 16;
// 1 = MN-major), N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, int b_mn_major) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(b_mn_major) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory descriptor of an MN-major tf32 operand in the 128-byte
// swizzle of 32-byte chunks: the fields of smem_desc_sw128 with layout type 1.
__device__ __forceinline__ uint64_t smem_desc_sw128_32b(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return (smem_desc_sw128(saddr, lbo_bytes, sbo_bytes) & ~(static_cast<uint64_t>(7) << 61)) |
         (static_cast<uint64_t>(1) << 61);
}

// Round to nearest tf32 (ties away from zero), as an fp32 bit pattern.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, uint64_t limit) {
  const bool ok = mbar_wait(bar, parity, limit);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(320, 1) attn_tf32_kernel(const __grid_constant__ Tf32Params p) {
  using C = TCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_BAR);
  uint64_t* bar_q = bars;
  uint64_t* bar_full = bars + 1;             // [NS] K or V tile landed
  uint64_t* bar_empty = bars + 1 + C::NS;    // [NS] slot read by the MMAs
  uint64_t* bar_s = bars + 1 + 2 * C::NS;    // [2] S of tile k ready in buffer k & 1
  uint64_t* bar_p = bar_s + 2;               // P_k written (128 arrivals)
  uint64_t* bar_pv = bar_p + 1;              // P_k V_k done
  uint64_t* bar_x = bar_pv + 1;              // [4] 64 arrivals: the two halves of 32 rows exchanged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_x + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.n_qt, qt = blockIdx.x % p.n_qt;
  const int L = p.L;
  const bool lab = p.label != nullptr && p.label[bh] == SVG_TEMPORAL;  // any other label: band 0
  const int G = lab ? p.G1 : p.G0, a = lab ? p.a1 : p.a0;
  const int q0 = qt * 128;
  const int q_last = min(q0 + 127, L - 1);
  // keys of the whole tile: [lo(q0), hi(q_last)); every row keeps its own key
  const int lo_cta = static_cast<int>(max(0LL, (static_cast<long long>(q0 / G) - a + 1) * G));
  const int hi_cta = static_cast<int>(min(static_cast<long long>(L), (static_cast<long long>(q_last / G) + a) * G));
  const int kt0 = lo_cta / 128;
  const int nk = (hi_cta + 127) / 128 - kt0;
  const HeadStrides& st = lab ? p.st_p : p.st_in;

  if (threadIdx.x == 0) {
    *abort_flag = (*reinterpret_cast<volatile int*>(p.status) & SVG_DEV_TIMEOUT) ? 1 : 0;
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_s[0], 1);
    mbar_init(&bar_s[1], 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_pv, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&bar_x[q], 64);
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool run = (*abort_flag == 0) && nk > 0;

  if (run && warp == 8 && lane == 0) {
    // ------------------------------------------------ TMA producer
    const CUtensorMap* tq = lab ? &p.tm_qp : &p.tm_q;
    const CUtensorMap* tk = lab ? &p.tm_kp : &p.tm_k;
    const CUtensorMap* tv = lab ? &p.tm_vp : &p.tm_v;
    tma_prefetch_desc(tq);
    tma_prefetch_desc(tk);
    tma_prefetch_desc(tv);
    const int th = st.tma_h(bh), tb = st.tma_b(bh);
    in_range(q0, L, p.status);
    mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
#pragma unroll
    for (int b = 0; b < C::BLOCKS; ++b) tma_load_4d(sQ + b * C::BLK_BYTES, tq, bar_q, b * 32, q0, th, tb);
    for (int n = 0; n < 2 * nk; ++n) {
      const int slot = n % C::NS;
      if (!mbar_wait(&bar_empty[slot], ((n / C::NS) & 1) ^ 1, p.wait_ns)) {
        *abort_flag = 1;
        atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
        break;
      }
      // entry n: K_0; K_{k+1} at 2k + 1; V_k at 2k + 2 (the last V at 2 nk - 1)
      const bool is_v = n > 0 && !((n & 1) && (n + 1) / 2 < nk);
      const int t = n == 0 ? 0 : !is_v ? (n + 1) / 2 : (n & 1) ? nk - 1 : n / 2 - 1;
      const CUtensorMap* tm = is_v ? tv : tk;
      const int row = (kt0 + t) * 128;
      in_range(row, L, p.status);
      mbar_arrive_expect_tx(&bar_full[slot], C::TILE_BYTES);
#pragma unroll
      for (int b = 0; b < C::BLOCKS; ++b)
        tma_load_4d(sRing + slot * C::TILE_BYTES + b * C::BLK_BYTES, tm, &bar_full[slot], b * 32, row, th, tb);
    }
  } else if (run && warp == 9) {
    // ------------------------------------------------ MMA issuer (whole warp; one elected lane issues)
    constexpr uint32_t idesc_qk = idesc_tf32(128, 128, 0);
    constexpr uint32_t idesc_pv = idesc_tf32(128, D, 1);
    const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
    const uint32_t ring = smem_u32(sRing);
    // S_j = Q K_j^T into buffer j & 1: K = 8 columns (32 bytes) per
    // instruction inside a 128-byte block, then the next block
    auto qk = [&](int j, int slot) {
      const uint64_t dk = smem_desc_sw128(ring + slot * C::TILE_BYTES, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 8; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * C::BLK_BYTES + (kk & 3) * 32) >> 4);
        ss_tf32(tmem + (j & 1) * 128, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
      }
      umma_commit_warp(&bar_s[j & 1]);
      umma_commit_warp(&bar_empty[slot]);
    };
    bool ok = wait_all(bar_q, 0, p.wait_ns) && wait_all(&bar_full[0], 0, p.wait_ns);
    if (ok) {
      tc_fence_after();
      qk(0, 0);
    }
    for (int k = 0; ok && k < nk; ++k) {
      // S_{k+1} goes into the other buffer, whose last reader (P_{k-1} V_{k-1})
      // was issued before it
      if (k + 1 < nk) {
        const int nK = 2 * k + 1, slotK = nK % C::NS;
        ok = wait_all(&bar_full[slotK], (nK / C::NS) & 1, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        qk(k + 1, slotK);
      }
      const int nV = (k + 1 < nk) ? 2 * k + 2 : 2 * nk - 1, slotV = nV % C::NS;
      ok = wait_all(bar_p, k & 1, p.wait_ns) && wait_all(&bar_full[slotV], (nV / C::NS) & 1, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      // O += P_k V_k: V MN-major (its 32-column blocks one BLK_BYTES apart,
      // 4-row atoms 512 bytes apart), 8 keys (two atoms, 1024 bytes) per
      // instruction
      const uint64_t dv = smem_desc_sw128_32b(ring + slotV * C::TILE_BYTES, C::BLK_BYTES, 512);
#pragma unroll
      for (int kk = 0; kk < 128 / 8; ++kk)
        ts_tf32(tmem + C::COL_O, tmem + (k & 1) * 128 + kk * 8, dv + static_cast<uint64_t>((kk * 1024) >> 4),
                idesc_pv, (k > 0 || kk > 0) ? 1u : 0u);
      umma_commit_warp(bar_pv);
      umma_commit_warp(&bar_empty[slotV]);
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
    }
  } else if (warp < 8) {
    // ------------------------------------------------ rows: softmax and epilogue
    const int q = warp & 3, h = warp >> 2;  // lane quarter; key half [64 h, 64 h + 64) of every tile
    const int r = q * 32 + lane;             // query row of the tile = TMEM lane
    const int x = q0 + r;
    const bool row_ok = x < L;
    int lo = 0, hi = 0;
    if (row_ok) {
      const long long g = x / G;
      lo = static_cast<int>(max(0LL, (g - a + 1) * G));
      hi = static_cast<int>(min(static_cast<long long>(L), (g + a) * G));
    }
    float* xm = reinterpret_cast<float*>(smem + C::SMEM_X);  // [2 parity][2 half][128 rows]
    float* fin = xm + 512;                                     // [2 half][128 rows] row sums
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t tO = trow + C::COL_O + h * (D / 2);  // this half's output columns
    float m = -INFINITY, l = 0.f;
    bool ok = run;
    for (int k = 0; ok && k < nk; ++k) {
      const uint32_t tS = trow + (k & 1) * 128 + h * 64;
      ok = wait_all(&bar_s[k & 1], (k >> 1) & 1, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[64];
      tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tmem_wait_ld();
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(v));  // no use before the wait
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(v + 32));
      const int y0 = (kt0 + k) * 128 + h * 64;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int y = y0 + c;
        const float sv = (y >= lo && y < hi) ? __uint_as_float(v[c]) * p.sl2 : -INFINITY;
        v[c] = __float_as_uint(sv);
        mx = fmaxf(mx, sv);
      }
      // the row's maximum over the whole tile, from both halves
      float* xk = xm + (k & 1) * 256;
      xk[h * 128 + r] = mx;
      mbar_arrive(&bar_x[q]);
      ok = wait_all(&bar_x[q], k & 1, p.wait_ns);
      if (!ok) break;
      const float m_new = fmaxf(m, fmaxf(mx, xk[(h ^ 1) * 128 + r]));
      // O holds P V of the earlier tiles once P_{k-1} V_{k-1} is done.  Waiting
      // for it every tile also keeps this tile's P arrival behind the MMA
      // warp's wait for the previous one (no two bar_p phases in flight).
      if (k > 0) {
        ok = wait_all(bar_pv, (k - 1) & 1, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
      }
      // rescale this half of O when the row's reference grew (both halves
      // take the same decision: same m, same m_new)
      const float alpha = (m_new == -INFINITY || m == m_new) ? 1.f : ex2_approx(m - m_new);
      if (__any_sync(0xffffffffu, k > 0 && alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[16];
          tmem_ld16(tO + c * 16, ov);
          tmem_wait_ld();
          reg_fence16(ov);
#pragma unroll
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st16(tO + c * 16, ov);
        }
      }
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float sv = __uint_as_float(v[c]);
        const float pr = (m_new == -INFINITY) ? 0.f : ex2_approx(sv - m_new);  // masked: exp2(-inf) = 0
        v[c] = to_tf32(pr);
        sum += __uint_as_float(v[c]);
      }
      l = l * alpha + sum;
      m = m_new;
      tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(v));
      tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(v + 32));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    // the row sum of both halves
    if (ok) {
      fin[h * 128 + r] = l;
      mbar_arrive(&bar_x[q]);
      ok = wait_all(&bar_x[q], nk & 1, p.wait_ns);
    }
    if (ok) ok = wait_all(bar_pv, (nk - 1) & 1, p.wait_ns);
    if (ok) {
      tc_fence_after();
      const float lt = fin[r] + fin[128 + r];
      const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
      const bool store_ok = row_ok && in_range(x, L, p.status) && in_range(bh, p.BH, p.status);
      float* out = (lab ? p.op : p.o) + st.head(store_ok ? bh : 0) + (store_ok ? x : 0) * st.sl + h * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[16];
        tmem_ld16(tO + c * 16, ov);
        tmem_wait_ld();
        reg_fence16(ov);
        if (store_ok) {
          float4* dst = reinterpret_cast<float4*>(out + c * 16);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l, __uint_as_float(ov[4 * e + 1]) * inv_l,
                                 __uint_as_float(ov[4 * e + 2]) * inv_l, __uint_as_float(ov[4 * e + 3]) * inv_l);
        }
      }
    } else if (run && lane == 0) {
      *abort_flag = 1;
      atomicOr(p.status, static_cast<int>(SVG_DEV_TIMEOUT));
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

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 4D view (d, row, head, batch entry) of an fp32 tensor laid out as s: boxes
// of 32 columns (128 bytes) x 128 rows in the given 128-byte swizzle.
svg_status make_tile_map_f32(CUtensorMap* map, const void* base, const HeadStrides& s, int L, int D,
                             CUtensorMapSwizzle swizzle) {
  static EncodeFn enc = nullptr;
  if (enc == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<EncodeFn>(ptr);
  }
  if (enc == nullptr) return fail(SVG_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(s.H),
                              static_cast<cuuint64_t>(s.nb)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.sl) * 4, static_cast<cuuint64_t>(s.sh) * 4,
                                 static_cast<cuuint64_t>(s.sb) * 4};
  const cuuint32_t box[4] = {32, 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SVG_ERR_CUDA, "cuTensorMapEncodeTiled (fp32) failed (%d)", static_cast<int>(r));
  return SVG_OK;
}

template <int D>
svg_status launch_tf32_d(const BandAttnArgs& a, cudaStream_t stream) {
  using C = TCfg<D>;
  Tf32Params p;
  memset(&p, 0, sizeof(p));
  const bool perm = a.label != nullptr;
  p.st_in = a.hs;
  p.st_p = perm ? a.hsp : a.hs;
  svg_status st;
  constexpr CUtensorMapSwizzle kmaj = CU_TENSOR_MAP_SWIZZLE_128B, mnmaj = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;
  if ((st = make_tile_map_f32(&p.tm_q, a.q, p.st_in, a.L, D, kmaj)) != SVG_OK) return st;
  if ((st = make_tile_map_f32(&p.tm_k, a.k, p.st_in, a.L, D, kmaj)) != SVG_OK) return st;
  if ((st = make_tile_map_f32(&p.tm_v, a.v, p.st_in, a.L, D, mnmaj)) != SVG_OK) return st;
  if ((st = make_tile_map_f32(&p.tm_qp, perm ? a.qp : a.q, p.st_p, a.L, D, kmaj)) != SVG_OK) return st;
  if ((st = make_tile_map_f32(&p.tm_kp, perm ? a.kp : a.k, p.st_p, a.L, D, kmaj)) != SVG_OK) return st;
  if ((st = make_tile_map_f32(&p.tm_vp, perm ? a.vp : a.v, p.st_p, a.L, D, mnmaj)) != SVG_OK) return st;
  p.o = static_cast<float*>(a.o);
  p.op = static_cast<float*>(perm ? a.op : a.o);
  p.label = a.label;
  p.BH = a.B * a.H;
  p.L = a.L;
  p.n_qt = (a.L + 127) / 128;
  p.G0 = a.G0;
  p.a0 = a.a0;
  p.G1 = a.G1;
  p.a1 = a.a1;
  p.sl2 = a.scale * 1.4426950408889634f;
  p.status = a.status;
  p.wait_ns = a.wait_ns;
  const long long grid = static_cast<long long>(p.BH) * p.n_qt;
  if (grid > 0x7fffffffLL) return fail(SVG_ERR_UNSUPPORTED, "grid too large");
  cudaError_t e = cudaFuncSetAttribute(attn_tf32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_check(e, "cudaFuncSetAttribute(tf32 attention smem)");
  attn_tf32_kernel<D><<<static_cast<unsigned>(grid), C::THREADS, C::SMEM_BYTES, stream>>>(p);
  return cuda_check(cudaGetLastError(), "tf32 attention launch");
}

}  // namespace

svg_status launch_attn_tf32(const BandAttnArgs& a, cudaStream_t stream) {
  if (a.modes != nullptr || a.fused || a.s2)
    return fail(SVG_ERR_UNSUPPORTED, "the tf32 kernel runs the spatial / temporal bands only");
  switch (a.d) {
    case 32: return launch_tf32_d<32>(a, stream);
    case 64: return launch_tf32_d<64>(a, stream);
    case 128: return launch_tf32_d<128>(a, stream);
    default: return fail(SVG_ERR_UNSUPPORTED, "tf32 attention supports d in {32, 64, 128}, got %d", a.d);
  }
}

}  // namespace svg
