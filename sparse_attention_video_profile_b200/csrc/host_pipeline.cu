// host_pipeline.cu -- svg_sparse_3d_attn_host: one whole sparse 3D-attention
// call on HOST buffers, with the host<->device copies overlapped with the
// computation.
//
// Every head is independent (its profiling, permutation and attention touch
// no other head), so the call is cut into chunks of heads.  Two device slots
// (from the caller's workspace) alternate between chunks:
//   copy-in stream   H2D of chunk c's q, k, v        (after slot c%2 is free)
//   caller's stream  the whole call on chunk c, with svg_sparse_3d_attn's
//                    choice of layout (fused into attention, or permute ->
//                    attention -> unpermute)
//   copy-out stream  D2H of chunk c's o, mse, label  (after its compute)
// so the copies of one chunk run under the kernels of its neighbours.  The
// results are bit-identical to svg_sparse_3d_attn on the same data.
#include <mutex>

#include "internal.h"

namespace svg {
namespace {

constexpr int kMaxDevices = 64;

struct PipeResources {
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_entry = nullptr, ev_in[2] = {nullptr, nullptr}, ev_done[2] = {nullptr, nullptr},
              ev_free[2] = {nullptr, nullptr};
  bool ready = false;
};

std::mutex g_pipe_mutex;
PipeResources g_pipe[kMaxDevices];
// Held by a call for its whole enqueue: the streams and events of a device
// are shared, so two host threads must not interleave their records and waits.
std::mutex g_enqueue_mutex[kMaxDevices];

// Streams and events of the current device, created on first use and kept.
svg_status pipe_resources(PipeResources** out, int* dev_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SVG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  PipeResources& r = g_pipe[dev];
  if (!r.ready) {
    const unsigned ef = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&r.s_in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&r.s_out, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&r.ev_entry, ef)) != cudaSuccess)
      return cuda_check(e, "pipeline stream/event creation");
    for (int i = 0; i < 2; ++i)
      if ((e = cudaEventCreateWithFlags(&r.ev_in[i], ef)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&r.ev_done[i], ef)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&r.ev_free[i], ef)) != cudaSuccess)
        return cuda_check(e, "pipeline event creation");
    r.ready = true;
  }
  *out = &r;
  return SVG_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct SlotLayout {
  size_t tensor;   // one chunk tensor [hc, L, d]
  size_t prof;     // profiling workspace of a chunk
  size_t mse, label, rows;
  size_t slot;     // bytes per slot
  int ntensors;
};

// Keys per profiling chunk of the whole call (all B*H heads): every chunk of
// heads splits its keys the same way, so its MSEs round exactly as the device
// call's.
int full_call_chunk(const svg_shape* s, int S) {
  ProfileLayout full;
  if (!profile_layout(s->B, s->H, s->N * s->F, s->d, s->dtype, S, &full)) return 0;
  return full.chunk;
}

SlotLayout slot_layout(const svg_shape* s, int S, int hc, bool fused) {
  SlotLayout l{};
  const size_t es = s->dtype == SVG_BF16 ? 2 : 4;
  l.tensor = align256(static_cast<size_t>(hc) * s->N * s->F * s->d * es);
  ProfileLayout pl;
  if (!profile_layout(1, hc, s->N * s->F, s->d, s->dtype, S, &pl, 0, full_call_chunk(s, S))) pl.total = 0;
  l.prof = align256(pl.total);
  l.mse = align256(static_cast<size_t>(hc) * 2 * sizeof(float));
  l.label = align256(static_cast<size_t>(hc));
  l.rows = align256(static_cast<size_t>(S) * sizeof(int32_t));
  l.ntensors = fused ? 4 : 8;  // q k v o (+ token-major copies unless the layout is fused)
  l.slot = l.ntensors * l.tensor + l.prof + l.mse + l.label + l.rows;
  return l;
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" {

SVG_API size_t svg_sparse_3d_attn_host_workspace_size(const svg_shape* shape, int32_t a2, int32_t S,
                                                      int32_t heads_per_chunk) {
  if (shape == nullptr || heads_per_chunk < 1 || S < 1 || S > 128 || a2 < 1) return 0;
  if (svg_profile_workspace_size(shape, S) == 0) return 0;
  const int hc = heads_per_chunk < shape->B * shape->H ? heads_per_chunk : shape->B * shape->H;
  return 2 * slot_layout(shape, S, hc, whole_call_fused(shape, a2)).slot;
}

SVG_API svg_status svg_sparse_3d_attn_host(const svg_shape* shape, const void* q_host, const void* k_host,
                                           const void* v_host, void* o_host, int32_t a1, int32_t a2,
                                           const int32_t* rows_host, int32_t S, float* mse_host, int8_t* label_host,
                                           int32_t heads_per_chunk, void* workspace, size_t workspace_bytes,
                                           int32_t* status_dev, void* stream) {
  if (shape == nullptr) return fail(SVG_ERR_INVALID_ARG, "shape is NULL");
  if (shape->layout != SVG_LAYOUT_BHLD)
    return fail(SVG_ERR_UNSUPPORTED, "the host-buffer call copies whole heads: [B, H, L, d] tensors only");
  if (!q_host || !k_host || !v_host || !o_host || !rows_host || !mse_host || !label_host || !workspace)
    return fail(SVG_ERR_INVALID_ARG, "NULL host buffer or workspace");
  if (heads_per_chunk < 1) return fail(SVG_ERR_INVALID_ARG, "heads_per_chunk must be >= 1");
  const size_t need = svg_sparse_3d_attn_host_workspace_size(shape, a2, S, heads_per_chunk);
  if (need == 0) return fail(SVG_ERR_INVALID_ARG, "bad shape, S or a2");
  if (workspace_bytes < need) return fail(SVG_ERR_WORKSPACE, "workspace %zu bytes < %zu required", workspace_bytes, need);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(SVG_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const int BH = shape->B * shape->H;
  const int hc = heads_per_chunk < BH ? heads_per_chunk : BH;
  const bool fused = whole_call_fused(shape, a2);
  const SlotLayout lay = slot_layout(shape, S, hc, fused);
  const size_t es = shape->dtype == SVG_BF16 ? 2 : 4;
  const size_t head_bytes = static_cast<size_t>(shape->N) * shape->F * shape->d * es;

  PipeResources* r = nullptr;
  int dev = 0;
  svg_status st = pipe_resources(&r, &dev);
  if (st != SVG_OK) return st;
  std::lock_guard<std::mutex> enqueue_lock(g_enqueue_mutex[dev]);
  const cudaStream_t sc = static_cast<cudaStream_t>(stream);
  cudaError_t e;
#define SVG_CU(call, what)                                   \
  do {                                                       \
    if ((e = (call)) != cudaSuccess) return cuda_check(e, what); \
  } while (0)
  // everything waits for the work already on the caller's stream
  SVG_CU(cudaEventRecord(r->ev_entry, sc), "event record");
  SVG_CU(cudaStreamWaitEvent(r->s_in, r->ev_entry, 0), "stream wait");
  SVG_CU(cudaStreamWaitEvent(r->s_out, r->ev_entry, 0), "stream wait");

  uint8_t* base = static_cast<uint8_t*>(workspace);
  const int n_chunks = (BH + hc - 1) / hc;
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c & 1;
    const int h0 = c * hc;
    const int nh = (h0 + hc <= BH) ? hc : BH - h0;
    uint8_t* slot = base + s * lay.slot;
    uint8_t *q = slot, *k = slot + lay.tensor, *v = slot + 2 * lay.tensor, *o = slot + 3 * lay.tensor;
    uint8_t *qp = slot + 4 * lay.tensor, *kp = slot + 5 * lay.tensor, *vp = slot + 6 * lay.tensor,
            *op = slot + 7 * lay.tensor;
    uint8_t* prof = slot + lay.ntensors * lay.tensor;
    float* mse = reinterpret_cast<float*>(prof + lay.prof);
    int8_t* lab = reinterpret_cast<int8_t*>(prof + lay.prof + lay.mse);
    int32_t* rows = reinterpret_cast<int32_t*>(prof + lay.prof + lay.mse + lay.label);
    const size_t off = static_cast<size_t>(h0) * head_bytes, bytes = static_cast<size_t>(nh) * head_bytes;
    // copy in (once slot s is free again)
    if (c >= 2) SVG_CU(cudaStreamWaitEvent(r->s_in, r->ev_free[s], 0), "stream wait");
    SVG_CU(cudaMemcpyAsync(q, static_cast<const uint8_t*>(q_host) + off, bytes, cudaMemcpyHostToDevice, r->s_in), "H2D");
    SVG_CU(cudaMemcpyAsync(k, static_cast<const uint8_t*>(k_host) + off, bytes, cudaMemcpyHostToDevice, r->s_in), "H2D");
    SVG_CU(cudaMemcpyAsync(v, static_cast<const uint8_t*>(v_host) + off, bytes, cudaMemcpyHostToDevice, r->s_in), "H2D");
    if (c < 2)
      SVG_CU(cudaMemcpyAsync(rows, rows_host, static_cast<size_t>(S) * sizeof(int32_t), cudaMemcpyHostToDevice, r->s_in),
             "H2D rows");
    SVG_CU(cudaEventRecord(r->ev_in[s], r->s_in), "event record");
    // compute on the caller's stream
    SVG_CU(cudaStreamWaitEvent(sc, r->ev_in[s], 0), "stream wait");
    svg_shape cs = *shape;
    cs.B = 1;
    cs.H = nh;
    if ((st = profile_heads_impl(&cs, shape_strides(&cs), q, k, v, a1, a2, rows, S, mse, lab, prof, lay.prof, status_dev, sc,
                                 full_call_chunk(shape, S))) != SVG_OK)
      return st;
    if (fused) {
      if ((st = svg_block_sparse_attn_fused(&cs, q, k, v, o, lab, a1, a2, status_dev, stream)) != SVG_OK) return st;
    } else {
      if ((st = svg_permute_qkv(&cs, q, k, v, qp, kp, vp, lab, stream)) != SVG_OK) return st;
      if ((st = svg_block_sparse_attn(&cs, q, k, v, qp, kp, vp, o, op, lab, a1, a2, status_dev, stream)) != SVG_OK)
        return st;
      if ((st = svg_unpermute(&cs, op, o, lab, stream)) != SVG_OK) return st;
    }
    SVG_CU(cudaEventRecord(r->ev_done[s], sc), "event record");
    // copy out
    SVG_CU(cudaStreamWaitEvent(r->s_out, r->ev_done[s], 0), "stream wait");
    SVG_CU(cudaMemcpyAsync(static_cast<uint8_t*>(o_host) + off, o, bytes, cudaMemcpyDeviceToHost, r->s_out), "D2H");
    SVG_CU(cudaMemcpyAsync(mse_host + 2 * h0, mse, static_cast<size_t>(nh) * 2 * sizeof(float), cudaMemcpyDeviceToHost,
                           r->s_out),
           "D2H mse");
    SVG_CU(cudaMemcpyAsync(label_host + h0, lab, static_cast<size_t>(nh), cudaMemcpyDeviceToHost, r->s_out), "D2H label");
    SVG_CU(cudaEventRecord(r->ev_free[s], r->s_out), "event record");
  }
  // the caller's stream resumes once every copy-out is done
  for (int s = 0; s < 2 && s < n_chunks; ++s) SVG_CU(cudaStreamWaitEvent(sc, r->ev_free[s], 0), "stream wait");
#undef SVG_CU
  return SVG_OK;
}

}  // extern "C"
