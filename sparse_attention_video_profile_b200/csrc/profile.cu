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
// Stage 1, bf16 (profile_sm100.cu): the key axis is split into chunks, one
// CTA per (chunk, head) holds all sampled rows as one 128-row tile, computes
// S = Q K^T on the tensor cores and keeps the three online-softmax states,
// with P V products into three TMEM accumulators.  Partial (max, sum,
// unnormalised output) triples go to the workspace.
// Stage 2 (profile_combine_rows_kernel, one block per sampled row and head;
// profile_finalize_kernel, one block per head): merges the chunk partials in
// a fixed order, forms O_d, O_s, O_t, and reduces the squared differences in
// fp64 with fixed trees -- so repeated calls return identical bits.
// fp32 inputs use profile_simt_kernel (one warp per row, all keys) for stage
// 1 and the same stage 2.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace svg {
namespace {

constexpr int kKT = 128;  // keys per tile of the bf16 stage 1

struct ProfParams {
  const void* q;  // q, k, v laid out as hs
  const void* k;
  const void* v;
  HeadStrides hs;
  const int32_t* rows;
  float* ws_o;   // [BH][nch][3][S_pad][D]
  float* ws_ml;  // [BH][nch][3][S_pad][2]  (max in log2 units, sum)
  int BH, L, N, F, S, S_pad, nch, chunk;
  int a1, a2;
  float sl2;
};

// fp32 stage 1: one warp per (head, sampled row, key chunk); the chunk
// partials go to the same workspace layout as the bf16 stage 1's.  The four
// rows of a block share each 32-key step's K and V rows, loaded once into
// shared memory with coalesced reads (K rows padded by one word, so lane j
// reading key j's column c hits bank (j + c) mod 32).
template <int D>
__global__ void __launch_bounds__(128) profile_simt_kernel(const ProfParams p) {
  constexpr int PER = D / 32;
  __shared__ float sq[4][D];
  __shared__ float sK[32][D + 1];
  __shared__ float sV[32][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x * 4 + warp;  // < S_pad: S_pad is a multiple of the block's 4 rows
  const int bh = blockIdx.y, ch = blockIdx.z;
  const int y_begin = ch * p.chunk, y_end = min(p.L, y_begin + p.chunk);
  const long long hoff = p.hs.head(bh), sl = p.hs.sl;
  const float* q = static_cast<const float*>(p.q) + hoff;
  const float* k = static_cast<const float*>(p.k) + hoff;
  const float* v = static_cast<const float*>(p.v) + hoff;
  const int x = min(max(p.rows[min(s, p.S - 1)], 0), p.L - 1);
  const int ir = x / p.F, jr = x % p.F;
  for (int c = lane; c < D; c += 32) sq[warp][c] = q[x * sl + c] * p.sl2;
  __syncwarp();
  float m[3], l[3], acc[3][PER];
#pragma unroll
  for (int vv = 0; vv < 3; ++vv) {
    m[vv] = -INFINITY;
    l[vv] = 0.f;
#pragma unroll
    for (int t = 0; t < PER; ++t) acc[vv][t] = 0.f;
  }
  for (int y0 = y_begin; y0 < y_end; y0 += 32) {
    __syncthreads();  // the previous step's rows are no longer read
    for (int e = threadIdx.x; e < 32 * D; e += 128) {
      const int r = e / D, c = e - r * D;
      const bool in = y0 + r < y_end;
      sK[r][c] = in ? k[(y0 + r) * sl + c] : 0.f;
      sV[r][c] = in ? v[(y0 + r) * sl + c] : 0.f;
    }
    __syncthreads();
    const int y = y0 + lane;
    float sc = -INFINITY;
    int iy = -1, jy = -1;
    if (y < y_end) {
      float dot = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) dot = fmaf(sq[warp][c], sK[lane][c], dot);
      sc = dot;
      iy = y / p.F;
      jy = y % p.F;
    }
    float pv[3];
#pragma unroll
    for (int vv = 0; vv < 3; ++vv) {
      bool ok = y < y_end;
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
    const int nvalid = min(32, y_end - y0);
    for (int jj = 0; jj < nvalid; ++jj) {
      float vals[PER];
#pragma unroll
      for (int t = 0; t < PER; ++t) vals[t] = sV[jj][lane + 32 * t];
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
    const size_t base = ((static_cast<size_t>(bh) * p.nch + ch) * 3 + vv) * p.S_pad + s;
#pragma unroll
    for (int t = 0; t < PER; ++t) p.ws_o[base * D + lane + 32 * t] = acc[vv][t];
    if (lane == 0) {
      p.ws_ml[base * 2 + 0] = m[vv];  // already in log2 units
      p.ws_ml[base * 2 + 1] = l[vv];
    }
  }
}

constexpr int kCombineThreads = 128;

// Stage 2a: one block per (sampled row, head).  Merges the chunk partials of
// the three outputs of that row (thread c owns column c) and reduces the
// row's squared differences (O_s - O_d)^2 and (O_t - O_d)^2 over d in a fixed
// order, in fp64.
__global__ void __launch_bounds__(kCombineThreads)
    profile_combine_rows_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_ml, int S_pad, int D,
                                int nch, double* __restrict__ part) {
  __shared__ double red[3][kCombineThreads / 32];
  const int s = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  double dsq = 0.0, dtq = 0.0, ddq = 0.0;
  if (c < D) {
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
    dsq = dsp * dsp;
    dtq = dtp * dtp;
    ddq = static_cast<double>(ov[0]) * ov[0];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dsq += __shfl_xor_sync(0xffffffffu, dsq, off);
    dtq += __shfl_xor_sync(0xffffffffu, dtq, off);
    ddq += __shfl_xor_sync(0xffffffffu, ddq, off);
  }
  if ((c & 31) == 0) {
    red[0][c >> 5] = dsq;
    red[1][c >> 5] = dtq;
    red[2][c >> 5] = ddq;
  }
  __syncthreads();
  if (c == 0) {
    double a = 0.0, b = 0.0, cc = 0.0;
#pragma unroll
    for (int w = 0; w < kCombineThreads / 32; ++w) {
      a += red[0][w];
      b += red[1][w];
      cc += red[2][w];
    }
    part[(static_cast<size_t>(bh) * S_pad + s) * 3 + 0] = a;
    part[(static_cast<size_t>(bh) * S_pad + s) * 3 + 1] = b;
    part[(static_cast<size_t>(bh) * S_pad + s) * 3 + 2] = cc;
  }
}

// Stage 2b: per head, sums the S rows' partial sums in a fixed order and
// writes the two MSEs and the label.
__global__ void __launch_bounds__(kCombineThreads)
    profile_finalize_kernel(const double* __restrict__ part, int S, int S_pad, int D, float* __restrict__ mse,
                            int8_t* __restrict__ label, const int* __restrict__ status, int* __restrict__ status_out) {
  __shared__ double red[2][kCombineThreads];
  const int bh = blockIdx.x;
  double a = 0.0, b = 0.0;
  for (int s = threadIdx.x; s < S; s += kCombineThreads) {
    a += part[(static_cast<size_t>(bh) * S_pad + s) * 3 + 0];
    b += part[(static_cast<size_t>(bh) * S_pad + s) * 3 + 1];
  }
  red[0][threadIdx.x] = a;
  red[1][threadIdx.x] = b;
  __syncthreads();
  for (int w = kCombineThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      red[0][threadIdx.x] += red[0][threadIdx.x + w];
      red[1][threadIdx.x] += red[1][threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double n = static_cast<double>(S) * D;
    const float ms = static_cast<float>(red[0][0] / n), mt = static_cast<float>(red[1][0] / n);
    const int bits = status != nullptr ? (*status & (SVG_DEV_TIMEOUT | SVG_DEV_RANGE | SVG_DEV_BOUNDS)) : 0;
    const bool failed = bits != 0;
    if (failed && status_out != nullptr && bh == 0) atomicOr(status_out, bits);
    mse[bh * 2 + 0] = failed ? __int_as_float(0x7fc00000) : ms;
    mse[bh * 2 + 1] = failed ? __int_as_float(0x7fc00000) : mt;
    label[bh] = failed ? static_cast<int8_t>(-1) : ((mt < ms) ? SVG_TEMPORAL : SVG_SPATIAL);
  }
}

// Sparse-vDiT mode selection, one block per head ("Sparse-vDiT" review,
// "What carries the argument" and the referee report on Sec. 4.2, Eq. (2)):
// for each sparse mode i (skip, diagonal, multi-diagonal, stripe),
//   L_i = MSE(O_i - O_dense) + lambda * (1 - S_i),
// S_i the mode's sparsity (the share of (query, key) pairs it does not
// compute; 1 for skip).  The mode with the smallest L_i wins unless every
// L_i exceeds epsilon, in which case the head keeps full attention.  The
// MSEs are over the sampled rows and d, like the online profiling's.
__global__ void __launch_bounds__(kCombineThreads)
    mode_search_kernel(const double* __restrict__ part1, const double* __restrict__ part2, int S, int S_pad, int D,
                       float4 sparsity, float lambda, float epsilon, float* __restrict__ loss,
                       int8_t* __restrict__ mode, const int* __restrict__ status) {
  __shared__ double red[4][kCombineThreads];
  const int bh = blockIdx.x;
  double sdiag = 0.0, smd = 0.0, sskip = 0.0, sstripe = 0.0;
  for (int s = threadIdx.x; s < S; s += kCombineThreads) {
    const size_t r = (static_cast<size_t>(bh) * S_pad + s) * 3;
    sdiag += part1[r + 0];
    smd += part1[r + 1];
    sskip += part1[r + 2];
    sstripe += part2[r + 0];
  }
  red[0][threadIdx.x] = sskip;
  red[1][threadIdx.x] = sdiag;
  red[2][threadIdx.x] = smd;
  red[3][threadIdx.x] = sstripe;
  __syncthreads();
  for (int w = kCombineThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w)
#pragma unroll
      for (int q = 0; q < 4; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double n = static_cast<double>(S) * D;
    const float sp[4] = {sparsity.x, sparsity.y, sparsity.z, sparsity.w};  // skip, diagonal, multi-diag, stripe
    const int modes[4] = {SVG_MODE_SKIP, SVG_MODE_DIAGONAL, SVG_MODE_MULTIDIAG, SVG_MODE_STRIPE};
    const bool failed = status != nullptr && (*status & (SVG_DEV_TIMEOUT | SVG_DEV_RANGE | SVG_DEV_BOUNDS));
    int best = -1;
    float best_l = 0.f;
    for (int q = 0; q < 4; ++q) {
      const float li = static_cast<float>(red[q][0] / n) + lambda * (1.f - sp[q]);
      loss[bh * 4 + q] = failed ? __int_as_float(0x7fc00000) : li;
      if (best < 0 || li < best_l) {
        best = q;
        best_l = li;
      }
    }
    mode[bh] = failed ? static_cast<int8_t>(-1)
                      : static_cast<int8_t>(best_l > epsilon ? SVG_MODE_FULL : modes[best]);
  }
}

template <int D>
svg_status launch_stage1_f32(const ProfParams& p, cudaStream_t stream) {
  if (p.nch > 65535) return fail(SVG_ERR_UNSUPPORTED, "%d key chunks exceed the grid limit", p.nch);
  dim3 grid((p.S_pad + 3) / 4, p.BH, p.nch);
  profile_simt_kernel<D><<<grid, 128, 0, stream>>>(p);
  return cuda_check(cudaGetLastError(), "fp32 profile launch");
}

// fp32 and tf32 tensors profile alike (fp32 on the CUDA cores)
int row_block(int /*d*/, int dtype) { return dtype == SVG_BF16 ? 128 : 4; }

}  // namespace

bool profile_layout(int B, int H, int L, int d, int dtype, int S, ProfileLayout* out, int max_chunks, int chunk_len) {
  if (B < 1 || H < 1 || L < 1 || S < 1 || S > 128 || max_chunks < 0 || chunk_len < 0) return false;
  const int rb = row_block(d, dtype);
  ProfileLayout lay{};
  lay.S_pad = (S + rb - 1) / rb * rb;
  if (dtype != SVG_BF16) {
    // fp32 (CUDA cores): enough key chunks for about 16 blocks of 4 rows per
    // SM, each chunk at least 1024 keys; chunk_len, when given, fixes it
    long long chunk;
    if (chunk_len > 0) {
      chunk = (static_cast<long long>(chunk_len) + 31) / 32 * 32;
    } else {
      const long long blocks = static_cast<long long>(B) * H * (lay.S_pad / 4);
      long long nch = (148LL * 16 + blocks - 1) / blocks;
      long long most = (L + 1023) / 1024;
      if (most > 65535) most = 65535;  // grid z
      if (nch > most) nch = most;
      if (max_chunks > 0 && nch > max_chunks) nch = max_chunks;
      if (nch < 1) nch = 1;
      chunk = ((L + nch - 1) / nch + 31) / 32 * 32;
    }
    if (chunk > L) chunk = L;
    lay.chunk = static_cast<int>(chunk);
    lay.n_chunks = static_cast<int>((L + chunk - 1) / chunk);
  } else if (chunk_len > 0) {
    long long chunk = (static_cast<long long>(chunk_len) + kKT - 1) / kKT * kKT;
    if (chunk > L) chunk = (L + kKT - 1) / kKT * kKT;
    lay.chunk = static_cast<int>(chunk);
    lay.n_chunks = static_cast<int>((L + chunk - 1) / chunk);
  } else {
    // One CTA per (chunk, head), one CTA per SM.  Pick the chunk count that
    // minimises waves x (key tiles per chunk + a fixed per-CTA cost of about
    // two tiles for setup, Q gather and the partials' store).
    const long long heads = static_cast<long long>(B) * H;
    const long long tiles = (L + kKT - 1) / kKT;
    long long limit = tiles;
    if (max_chunks > 0 && limit > max_chunks) limit = max_chunks;
    long long nch = 1, best = -1;
    for (long long c = 1; c <= limit && c <= 4096; ++c) {
      const long long waves = (heads * c + 147) / 148;
      const long long cost = waves * ((tiles + c - 1) / c + 2);
      if (best < 0 || cost < best) {
        best = cost;
        nch = c;
      }
    }
    long long chunk = (L + nch - 1) / nch;
    chunk = (chunk + kKT - 1) / kKT * kKT;
    lay.chunk = static_cast<int>(chunk);
    lay.n_chunks = static_cast<int>((L + chunk - 1) / chunk);
  }
  const size_t rows_total = static_cast<size_t>(B) * H * lay.n_chunks * 3 * lay.S_pad;
  lay.o_bytes = (rows_total * d * sizeof(float) + 255) / 256 * 256;
  lay.ml_bytes = (rows_total * 2 * sizeof(float) + 255) / 256 * 256;
  lay.part_bytes = (static_cast<size_t>(B) * H * lay.S_pad * 3 * sizeof(double) + 255) / 256 * 256;
  lay.status_bytes = 256;
  lay.total = lay.o_bytes + lay.ml_bytes + lay.part_bytes + lay.status_bytes;
  *out = lay;
  return true;
}

svg_status launch_profile_pass(int B, int H, int N, int F, int d, int dtype, float scale, const void* q,
                               const void* k, const void* v, const HeadStrides& hs, const int (&kind)[2], const int (&par)[2],
                               const int32_t* rows, int S, void* ws, const ProfileLayout& lay, double* part,
                               int* status, cudaStream_t stream) {
  ProfParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.hs = hs;
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
  p.a1 = par[0];
  p.a2 = par[1];
  p.sl2 = scale * 1.4426950408889634f;
  if (p.BH > 65535) return fail(SVG_ERR_UNSUPPORTED, "B*H = %d exceeds the grid limit", p.BH);
  svg_status st;
  if (dtype == SVG_BF16) {
    st = launch_profile_sm100(p.BH, N, F, d, scale, q, k, v, hs, kind, par, rows, S, p.ws_o, p.ws_ml, lay.n_chunks,
                              lay.chunk, status, stream);
  } else {
    if (kind[0] != kProfFrameBand || kind[1] != kProfPositionBand)
      return fail(SVG_ERR_UNSUPPORTED, "fp32 profiling supports the spatial / temporal pair only");
    if (d == 32) st = launch_stage1_f32<32>(p, stream);
    else if (d == 64) st = launch_stage1_f32<64>(p, stream);
    else if (d == 128) st = launch_stage1_f32<128>(p, stream);
    else return fail(SVG_ERR_UNSUPPORTED, "fp32 profiling supports d in {32, 64, 128}, got %d", d);
  }
  if (st != SVG_OK) return st;
  profile_combine_rows_kernel<<<dim3(S, p.BH), kCombineThreads, 0, stream>>>(p.ws_o, p.ws_ml, lay.S_pad, d,
                                                                              lay.n_chunks, part);
  return cuda_check(cudaGetLastError(), "profile combine launch");
}

static svg_status call_status_word(void* ws, const ProfileLayout& lay, int** out, cudaStream_t stream) {
  int* w = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + profile_status_offset(lay));
  cudaError_t e = cudaMemsetAsync(w, 0, sizeof(int), stream);
  if (e != cudaSuccess) return cuda_check(e, "cudaMemsetAsync(profiling status)");
  *out = w;
  return SVG_OK;
}

svg_status launch_profile(int B, int H, int N, int F, int d, int dtype, float scale, const void* q,
                          const void* k, const void* v, const HeadStrides& hs, int a1, int a2, const int32_t* rows, int S,
                          float* mse, int8_t* label, void* ws, const ProfileLayout& lay,
                          int* status_out, cudaStream_t stream) {
  int* status = nullptr;
  svg_status st = call_status_word(ws, lay, &status, stream);
  if (st != SVG_OK) return st;
  double* part = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + lay.o_bytes + lay.ml_bytes);
  const int kind[2] = {kProfFrameBand, kProfPositionBand}, par[2] = {a1, a2};
  if ((st = launch_profile_pass(B, H, N, F, d, dtype, scale, q, k, v, hs, kind, par, rows, S, ws, lay, part, status,
                                stream)) != SVG_OK)
    return st;
  profile_finalize_kernel<<<B * H, kCombineThreads, 0, stream>>>(part, S, lay.S_pad, d, mse, label, status,
                                                                   status_out);
  return cuda_check(cudaGetLastError(), "profile finalize launch");
}

svg_status launch_mode_search(int B, int H, int N, int F, int d, float scale, const void* q, const void* k,
                              const void* v, const HeadStrides& hs, const int32_t* rows, int S, int window, int md_half, int stripe,
                              float lambda, float epsilon, float* loss, int8_t* mode, void* ws,
                              const ProfileLayout& lay, double* part2, cudaStream_t stream) {
  int* status = nullptr;
  svg_status st = call_status_word(ws, lay, &status, stream);
  if (st != SVG_OK) return st;
  double* part1 = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + lay.o_bytes + lay.ml_bytes);
  const int kind1[2] = {kProfWindow, kProfPositionBand}, par1[2] = {window, md_half + 1};
  const int kind2[2] = {kProfPrefix, kProfNone}, par2[2] = {stripe, 0};
  if ((st = launch_profile_pass(B, H, N, F, d, SVG_BF16, scale, q, k, v, hs, kind1, par1, rows, S, ws, lay, part1,
                                status, stream)) != SVG_OK)
    return st;
  if ((st = launch_profile_pass(B, H, N, F, d, SVG_BF16, scale, q, k, v, hs, kind2, par2, rows, S, ws, lay, part2,
                                status, stream)) != SVG_OK)
    return st;
  // sparsity of each mode: 1 - kept pairs / L^2 (closed forms of the masks)
  const double L = static_cast<double>(N) * F;
  const double W = window < L - 1 ? window : L - 1;
  const double a = (md_half + 1 < F) ? md_half + 1 : F;
  const double Pn = stripe < L ? stripe : L;
  const double diag_pairs = L * (2 * W + 1) - W * (W + 1);
  const double md_pairs = static_cast<double>(N) * N * (F * (2 * a - 1) - a * (a - 1));
  const float4 sparsity = make_float4(1.f, static_cast<float>(1.0 - diag_pairs / (L * L)),
                                      static_cast<float>(1.0 - md_pairs / (L * L)), static_cast<float>(1.0 - Pn / L));
  mode_search_kernel<<<B * H, kCombineThreads, 0, stream>>>(part1, part2, S, lay.S_pad, d, sparsity, lambda, epsilon,
                                                            loss, mode, status);
  return cuda_check(cudaGetLastError(), "mode search launch");
}

}  // namespace svg
