// profile_noalloc.cu -- svg_profile_heads_noalloc: online profiling for
// callers that cannot allocate device memory.
//
// svg_profile_heads needs a caller-provided workspace for the per-chunk
// partial results.  Some callers have no way to provide one: a plugin whose
// host framework hands it only its input and output tensors, or a control
// loop that must never call cudaMalloc because that call can synchronise the
// whole device and stall every other stream at an unpredictable moment.
// This entry point gives them profiling with no allocation at all: its
// scratch is a fixed array in this library's device image, created once per
// device when the module loads and kept until the process exits.
#include <math.h>

#include <mutex>

#include "internal.h"

namespace svg {
namespace {

// The scratch array.  Host code must never pass `g_profile_scratch` itself
// to a kernel: on the host that name is only a stand-in for the symbol, not
// a device address.  Its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_profile_scratch[SVG_PROFILE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the lookup also loads this module on that device).
svg_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SVG_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_profile_scratch);
    if (e != cudaSuccess) return cuda_check(e, "cudaGetSymbolAddress(profile scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SVG_OK;
}

}  // namespace
}  // namespace svg

using namespace svg;

extern "C" SVG_API svg_status svg_profile_heads_noalloc(const svg_shape* shape, const void* q, const void* k,
                                                        const void* v, int32_t a1, int32_t a2, const int32_t* rows,
                                                        int32_t S, float* mse, int8_t* label, void* stream) {
  // argument checks (the same rules as svg_profile_heads)
  if (shape == nullptr) return fail(SVG_ERR_INVALID_ARG, "shape is NULL");
  if (shape->B < 1 || shape->H < 1 || shape->N < 1 || shape->F < 1 || shape->d < 1)
    return fail(SVG_ERR_INVALID_ARG, "B, H, N, F, d must be >= 1");
  if (static_cast<long long>(shape->N) * shape->F > (1LL << 30)) return fail(SVG_ERR_INVALID_ARG, "L too large");
  if (shape->dtype != SVG_BF16 && shape->dtype != SVG_FP32 && shape->dtype != SVG_TF32)
    return fail(SVG_ERR_INVALID_ARG, "unknown dtype");
  if (shape->layout != SVG_LAYOUT_BHLD && shape->layout != SVG_LAYOUT_BLHD)
    return fail(SVG_ERR_INVALID_ARG, "unknown layout");
  if (!(shape->scale >= 0.f) || isinf(shape->scale)) return fail(SVG_ERR_INVALID_ARG, "bad scale");
  if ((shape->dtype == SVG_BF16 && shape->d != 64 && shape->d != 128) ||
      (shape->dtype != SVG_BF16 && shape->d != 32 && shape->d != 64 && shape->d != 128))
    return fail(SVG_ERR_UNSUPPORTED, "unsupported head dim %d for this dtype", shape->d);
  for (const void* t : {q, k, v})
    if (t == nullptr || (reinterpret_cast<uintptr_t>(t) & 15u) != 0)
      return fail(SVG_ERR_INVALID_ARG, "q, k, v must be non-NULL and 16-byte aligned");
  if (!rows || !mse || !label) return fail(SVG_ERR_INVALID_ARG, "NULL rows/mse/label");
  if (a1 < 1 || a2 < 1) return fail(SVG_ERR_INVALID_ARG, "a1 and a2 must be >= 1");
  const int L = shape->N * shape->F;
  if (S < 1 || S > 128 || S > L) return fail(SVG_ERR_INVALID_ARG, "S must be in [1, min(128, L)], got %d", S);

  ProfileLayout lay;
  profile_layout(shape->B, shape->H, L, shape->d, shape->dtype, S, &lay);
  constexpr size_t kMax = SVG_PROFILE_NOALLOC_SCRATCH_BYTES;
  if (lay.total > kMax) {
    // Fewer, longer key chunks need less scratch.
    ProfileLayout one;
    profile_layout(shape->B, shape->H, L, shape->d, shape->dtype, S, &one, 1);
    const size_t per_chunk = one.o_bytes + one.ml_bytes;  // bytes that scale with the chunk count
    const long long fit = static_cast<long long>((kMax - one.part_bytes - one.status_bytes - 512) / per_chunk);
    if (one.total > kMax || fit < 1)
      return fail(SVG_ERR_WORKSPACE,
                  "profiling this shape needs at least %zu bytes of scratch, more than the %zu-byte static "
                  "array of svg_profile_heads_noalloc; use svg_profile_heads with a workspace",
                  one.total, kMax);
    profile_layout(shape->B, shape->H, L, shape->d, shape->dtype, S, &lay, static_cast<int>(fit));
    if (lay.total > kMax) return fail(SVG_ERR_WORKSPACE, "scratch layout does not fit the static array");
  }
  void* scratch = nullptr;
  svg_status st = scratch_address(&scratch);
  if (st != SVG_OK) return st;
  const float scale = shape->scale > 0.f ? shape->scale : 1.0f / sqrtf(static_cast<float>(shape->d));
  const int a1c = a1 < shape->N ? a1 : shape->N;
  const int a2c = a2 < shape->F ? a2 : shape->F;
  // the same kernels as svg_profile_heads, on the static scratch
  return launch_profile(shape->B, shape->H, shape->N, shape->F, shape->d, shape->dtype, scale, q, k, v,
                        shape_strides(shape), a1c, a2c,
                        rows, S, mse, label, scratch, lay, nullptr, static_cast<cudaStream_t>(stream));
}
