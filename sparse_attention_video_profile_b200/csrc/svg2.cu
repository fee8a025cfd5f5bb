// svg2.cu -- the data movement and selection steps of SVG2-style sparse
// attention (SVG2 explainer, section 2.A "Semantic-Aware Permutation" and
// 2.B "Centroid-Based Top-p Selection"), given each token's cluster:
//
//   svg2_sort       stable counting sort of a head's rows by cluster: the
//                   permutation (permuted position -> original row), each
//                   permuted row's cluster, and the cluster offsets;
//   svg2_gather     rows of Q / K / V moved to permuted order;
//   svg2_centroids  each cluster's mean, summed over its contiguous permuted
//                   rows in a fixed order (deterministic);
//   svg2_topp       per query cluster: key-cluster masses n_k exp(scale
//                   mu_q . mu_k) normalised, sorted (mass descending, index
//                   ascending), the shortest prefix reaching p kept, written
//                   as a bitmask over key clusters.
//
// Everything is deterministic: the histogram uses integer atomics only, the
// scatter ranks rows in their original order, and every floating-point sum
// runs in a fixed order.
#include <cuda_bf16.h>

#include "internal.h"

namespace svg {
namespace {

constexpr int kSortRows = 2048;  // rows per sort block

// Histogram of one block of rows: hist[bh][c][blk].
__global__ void __launch_bounds__(256) svg2_hist_kernel(const int32_t* __restrict__ assign, int L, int C, int nblk,
                                                        int32_t* __restrict__ hist, int* status) {
  extern __shared__ int32_t sh[];
  const int blk = blockIdx.x, bh = blockIdx.y;
  for (int c = threadIdx.x; c < C; c += blockDim.x) sh[c] = 0;
  __syncthreads();
  const int r0 = blk * kSortRows, r1 = min(L, r0 + kSortRows);
  const int32_t* a = assign + static_cast<size_t>(bh) * L;
  bool bad = false;
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    int c = a[r];
    if (c < 0 || c >= C) {
      bad = true;
      c = 0;
    }
    atomicAdd(&sh[c], 1);
  }
  if (bad) atomicOr(status, SVG_DEV_RANGE);
  __syncthreads();
  int32_t* hrow = hist + static_cast<size_t>(bh) * C * nblk;
  for (int c = threadIdx.x; c < C; c += blockDim.x) hrow[static_cast<size_t>(c) * nblk + blk] = sh[c];
}

// Exclusive scan of hist[bh] (cluster-major, block-minor) in place; off[bh][c]
// = first permuted position of cluster c, off[bh][C] = L.
__global__ void __launch_bounds__(1024) svg2_scan_kernel(int32_t* __restrict__ hist, int C, int nblk, int L,
                                                         int32_t* __restrict__ off) {
  __shared__ int32_t part[1024];
  const int bh = blockIdx.x, t = threadIdx.x;
  int32_t* h = hist + static_cast<size_t>(bh) * C * nblk;
  const int n = C * nblk;
  const int per = (n + 1023) / 1024;
  const int i0 = min(n, t * per), i1 = min(n, i0 + per);
  int32_t s = 0;
  for (int i = i0; i < i1; ++i) s += h[i];
  part[t] = s;
  __syncthreads();
  for (int w = 1; w < 1024; w <<= 1) {  // inclusive scan of the per-thread sums
    const int32_t v = t >= w ? part[t - w] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  int32_t run = part[t] - s;
  for (int i = i0; i < i1; ++i) {
    const int32_t v = h[i];
    h[i] = run;
    if (i % nblk == 0) off[static_cast<size_t>(bh) * (C + 1) + i / nblk] = run;
    run += v;
  }
  if (t == 0) off[static_cast<size_t>(bh) * (C + 1) + C] = L;
}

// One warp per block of rows: scatters the block's rows, in their original
// order, to their permuted positions.
__global__ void __launch_bounds__(32) svg2_scatter_kernel(const int32_t* __restrict__ assign, const int32_t* __restrict__ hist,
                                                          int L, int C, int nblk, int32_t* __restrict__ perm,
                                                          int32_t* __restrict__ cid) {
  extern __shared__ int32_t cnt[];
  const int blk = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
  const int32_t* h = hist + static_cast<size_t>(bh) * C * nblk;
  for (int c = lane; c < C; c += 32) cnt[c] = h[static_cast<size_t>(c) * nblk + blk];
  __syncwarp();
  const int r0 = blk * kSortRows, r1 = min(L, r0 + kSortRows);
  const int32_t* a = assign + static_cast<size_t>(bh) * L;
  int32_t* pm = perm + static_cast<size_t>(bh) * L;
  int32_t* ci = cid + static_cast<size_t>(bh) * L;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = r0; base < r1; base += 32) {
    const int r = base + lane;
    const bool act = r < r1;
    const unsigned active = __ballot_sync(0xffffffffu, act);
    int c = act ? a[r] : -1;
    if (act && (c < 0 || c >= C)) c = 0;  // reported by the histogram pass
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    if (act) {
      const int pos = cnt[c] + __popc(peers & lt);
      pm[pos] = r;
      ci[pos] = c;
    }
    __syncwarp();
    if (act && (peers & active & lt) == 0) cnt[c] += __popc(peers & active);
    __syncwarp();
  }
}

// Row gather: dst[bh][r] = src[bh][perm[bh][r]], rows of `rc` 16-byte chunks;
// dst is [BH, L, rc], src laid out as ss (strides in chunks).
__global__ void __launch_bounds__(256) svg2_gather_kernel(const uint4* __restrict__ src, const HeadStrides ss,
                                                          const int32_t* __restrict__ perm, uint4* __restrict__ dst,
                                                          int L, int rc, long long total) {
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = e / rc;  // bh * L + r
    const int c = static_cast<int>(e - row * rc);
    const int bh = static_cast<int>(row / L);
    __stcs(dst + e, __ldg(src + ss.head(bh) + perm[row] * ss.sl + c));
  }
}

// Four warps per (cluster, head): fp32 mean of the cluster's permuted rows;
// warp w sums rows w, w + 4, ... and the partial sums are added in warp
// order (deterministic).
template <int D>
__global__ void __launch_bounds__(128) svg2_centroid_kernel(const __nv_bfloat16* __restrict__ xp,
                                                            const int32_t* __restrict__ off, int L, int C,
                                                            float* __restrict__ mu) {
  constexpr int PER = D / 32;
  __shared__ float part[4][D];
  const int c = blockIdx.x, bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* o = off + static_cast<size_t>(bh) * (C + 1);
  const int r0 = o[c], r1 = o[c + 1];
  float s[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) s[e] = 0.f;
  const __nv_bfloat16* x = xp + static_cast<size_t>(bh) * L * D;
  for (int r = r0 + warp; r < r1; r += 4)
#pragma unroll
    for (int e = 0; e < PER; ++e) s[e] += __bfloat162float(x[static_cast<size_t>(r) * D + e * 32 + lane]);
#pragma unroll
  for (int e = 0; e < PER; ++e) part[warp][e * 32 + lane] = s[e];
  __syncthreads();
  if (warp != 0) return;
  const float inv = r1 > r0 ? 1.f / static_cast<float>(r1 - r0) : 0.f;
  float* m = mu + (static_cast<size_t>(bh) * C + c) * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int col = e * 32 + lane;
    m[col] = (((part[0][col] + part[1][col]) + part[2][col]) + part[3][col]) * inv;
  }
}

// One CTA per (query cluster, head): the kept key clusters as a bitmask.
template <int D>
__global__ void __launch_bounds__(256) svg2_topp_kernel(const float* __restrict__ mu_q, const float* __restrict__ mu_k,
                                                        const int32_t* __restrict__ off_k, int Cq, int Ck, int Ck_pad,
                                                        int W, float scale, float p, uint32_t* __restrict__ sel) {
  __shared__ float qv[D];
  __shared__ unsigned long long key[1024];  // (mass bits << 32) | ~index: sorts mass desc, index asc
  __shared__ float red[256];
  __shared__ uint32_t bits[32];
  const int cq = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const float* q = mu_q + (static_cast<size_t>(bh) * Cq + cq) * D;
  for (int e = t; e < D; e += 256) qv[e] = q[e];
  if (t < 32) bits[t] = 0u;
  __syncthreads();
  const int32_t* ok = off_k + static_cast<size_t>(bh) * (Ck + 1);
  // logits and their max over non-empty clusters
  float lmax = -INFINITY;
  for (int j = t; j < Ck; j += 256) {
    const float* kv = mu_k + (static_cast<size_t>(bh) * Ck + j) * D;
    float dot = 0.f;
    for (int e = 0; e < D; ++e) dot = fmaf(qv[e], kv[e], dot);
    const float lg = scale * dot;
    const int n = ok[j + 1] - ok[j];
    reinterpret_cast<float*>(key)[2 * j] = lg;  // scratch: logit at the low word of key[j]
    if (n > 0) lmax = fmaxf(lmax, lg);
  }
  red[t] = lmax;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (t < w) red[t] = fmaxf(red[t], red[t + w]);
    __syncthreads();
  }
  const float gmax = red[0];
  __syncthreads();
  float part = 0.f;
  for (int j = t; j < Ck_pad; j += 256) {
    float wj = 0.f;
    if (j < Ck) {
      const int n = ok[j + 1] - ok[j];
      const float lg = reinterpret_cast<float*>(key)[2 * j];
      wj = n > 0 ? static_cast<float>(n) * __expf(lg - gmax) : 0.f;
    }
    part += wj;
    key[j] = (static_cast<unsigned long long>(__float_as_uint(wj)) << 32) | (0xffffffffu - static_cast<uint32_t>(j));
  }
  red[t] = part;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (t < w) red[t] += red[t + w];
    __syncthreads();
  }
  const float total = red[0];
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= Ck_pad; k <<= 1)
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = t; i < Ck_pad; i += 256) {
        const int l = i ^ j;
        if (l > i) {
          const bool desc = (i & k) == 0;
          const unsigned long long a = key[i], b = key[l];
          if (desc ? a < b : a > b) {
            key[i] = b;
            key[l] = a;
          }
        }
      }
      __syncthreads();
    }
  // shortest prefix whose normalised mass reaches p (one thread, in order)
  if (t == 0) {
    const float target = p * total;
    float acc = 0.f;
    for (int i = 0; i < Ck_pad; ++i) {
      const float wj = __uint_as_float(static_cast<uint32_t>(key[i] >> 32));
      if (!(wj > 0.f)) break;
      const int j = static_cast<int>(0xffffffffu - static_cast<uint32_t>(key[i] & 0xffffffffu));
      bits[j >> 5] |= 1u << (j & 31);
      acc += wj;
      if (acc >= target) break;
    }
  }
  __syncthreads();
  uint32_t* out = sel + (static_cast<size_t>(bh) * Cq + cq) * W;
  for (int w = t; w < W; w += 256) out[w] = bits[w];
}

}  // namespace

Svg2Sizes svg2_sizes(int BH, int L, int Cq, int Ck, int d) {
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  Svg2Sizes z{};
  z.nblk = (L + kSortRows - 1) / kSortRows;
  z.W = (Ck + 31) / 32;
  const size_t rows = static_cast<size_t>(BH) * L;
  z.hist = al(static_cast<size_t>(BH) * (Cq > Ck ? Cq : Ck) * z.nblk * 4);
  z.perm = al(rows * 4);
  z.off_q = al(static_cast<size_t>(BH) * (Cq + 1) * 4);
  z.off_k = al(static_cast<size_t>(BH) * (Ck + 1) * 4);
  z.mu_q = al(static_cast<size_t>(BH) * Cq * d * 4);
  z.mu_k = al(static_cast<size_t>(BH) * Ck * d * 4);
  z.tensor = al(rows * d * 2);
  // hist (shared by the two sorts), perm_q, cid_q, perm_k, cid_k, offsets, centroids, Qp, Kp, Vp
  z.total = z.hist + 4 * z.perm + z.off_q + z.off_k + z.mu_q + z.mu_k + 3 * z.tensor;
  return z;
}

svg_status svg2_sort(const int32_t* assign, int BH, int L, int C, int nblk, int32_t* hist, int32_t* perm,
                     int32_t* cid, int32_t* off, int* status, cudaStream_t stream) {
  const size_t sh = static_cast<size_t>(C) * 4;
  svg2_hist_kernel<<<dim3(nblk, BH), 256, sh, stream>>>(assign, L, C, nblk, hist, status);
  svg2_scan_kernel<<<BH, 1024, 0, stream>>>(hist, C, nblk, L, off);
  svg2_scatter_kernel<<<dim3(nblk, BH), 32, sh, stream>>>(assign, hist, L, C, nblk, perm, cid);
  return cuda_check(cudaGetLastError(), "cluster sort launch");
}

svg_status svg2_gather(const void* src, const HeadStrides& ss, const int32_t* perm, void* dst, int BH, int L, int d,
                       cudaStream_t stream) {
  const int rc = d * 2 / 16;
  HeadStrides sc = ss;  // element strides -> 16-byte chunks (multiples of d)
  sc.sb /= 8;
  sc.sh /= 8;
  sc.sl /= 8;
  const long long total = static_cast<long long>(BH) * L * rc;
  const long long blocks = (total + 255) / 256;
  const unsigned grid = static_cast<unsigned>(blocks < 148LL * 64 ? blocks : 148LL * 64);
  svg2_gather_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(src), sc, perm, static_cast<uint4*>(dst), L,
                                               rc, total);
  return cuda_check(cudaGetLastError(), "cluster gather launch");
}

svg_status svg2_centroids(const void* xp, const int32_t* off, int BH, int L, int C, int d, float* mu,
                          cudaStream_t stream) {
  if (d == 128)
    svg2_centroid_kernel<128><<<dim3(C, BH), 128, 0, stream>>>(static_cast<const __nv_bfloat16*>(xp), off, L, C, mu);
  else
    svg2_centroid_kernel<64><<<dim3(C, BH), 128, 0, stream>>>(static_cast<const __nv_bfloat16*>(xp), off, L, C, mu);
  return cuda_check(cudaGetLastError(), "centroid launch");
}

svg_status svg2_topp(const float* mu_q, const float* mu_k, const int32_t* off_k, int BH, int Cq, int Ck, int d,
                     float scale, float p, uint32_t* sel, cudaStream_t stream) {
  int pad = 1;
  while (pad < Ck) pad <<= 1;
  const int W = (Ck + 31) / 32;
  if (d == 128)
    svg2_topp_kernel<128><<<dim3(Cq, BH), 256, 0, stream>>>(mu_q, mu_k, off_k, Cq, Ck, pad, W, scale, p, sel);
  else
    svg2_topp_kernel<64><<<dim3(Cq, BH), 256, 0, stream>>>(mu_q, mu_k, off_k, Cq, Ck, pad, W, scale, p, sel);
  return cuda_check(cudaGetLastError(), "top-p launch");
}

}  // namespace svg
