// Layer preparation without a caller-provided workspace.
//
// Some callers cannot allocate device memory: a host framework whose memory
// manager owns every device allocation (a pool or a fixed budget handed out at
// start-up), or a latency-critical loop in which cudaMalloc, which may
// synchronize the device, is not allowed. intlora_gen_aux needs a small
// scratch buffer (the per-CTA partial sums of the sigma reductions); this entry
// point takes that scratch from a fixed array compiled into the library
// instead, so the caller passes only inputs and outputs.
//
// The array lives in device memory of every GPU that loads the library, for
// the life of the process. Its size bounds the layers this entry point
// accepts (INTLORA_NOALLOC_MAX_ELEMENTS weight elements). Every call uses the
// same array: calls whose work overlaps on the GPU (different streams, no
// ordering between them) race on it and must be serialized by the caller.
// Nothing in the array has to start at zero: each statistics CTA overwrites
// its own partial before the finalize kernel reads it, so a call never sees
// the previous call's contents.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "intlora.h"
#include "intlora_kernels.h"

namespace {

// The statistics pass gives each CTA kStatsElementsPerCta (65,536) elements
// and one partial of kStatsPartialBytes (four fp64 sums, 32 bytes), so a layer
// of INTLORA_NOALLOC_MAX_ELEMENTS (4,194,304) elements needs 64 partials,
// 2 KB rounded to 256 bytes. The array holds 16 KB: room for 512 partials.
constexpr size_t kScratchBytes = 16384;
static_assert(((INTLORA_NOALLOC_MAX_ELEMENTS + intlora::kStatsElementsPerCta - 1) / intlora::kStatsElementsPerCta) *
                      intlora::kStatsPartialBytes <= kScratchBytes,
              "the built-in scratch must hold the partials of the largest layer this entry point accepts");
static __device__ __align__(256) double g_scratch[kScratchBytes / sizeof(double)];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device. In host code g_scratch
// names a host-side stand-in, not device memory, so the address is looked up
// once per device (with that device current) and cached.
cudaError_t scratch_on_current_device(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" intlora_status intlora_gen_aux_noalloc(const float* W, int64_t d, int64_t n,
                                                  uint64_t seed, uint32_t stream_id, float alpha,
                                                  int32_t w_bits, double* sigma_w_out,
                                                  double* sigma_r_out, float* r_star_out,
                                                  void* w_round_out, int64_t ld_w_out,
                                                  float* s_out, int32_t* z_out, void* stream) {
  // Arguments first, through the regular entry point with no workspace: it
  // returns INTLORA_ERR_INVALID_ARG for bad arguments and otherwise reports the
  // missing workspace without launching anything.
  intlora_status st = intlora_gen_aux(W, d, n, seed, stream_id, alpha, w_bits, sigma_w_out,
                                      sigma_r_out, r_star_out, w_round_out, ld_w_out, s_out, z_out,
                                      nullptr, 0, stream);
  if (st != INTLORA_ERR_WORKSPACE) return st;
  char msg[200];
  if (d > INTLORA_NOALLOC_MAX_ELEMENTS / n) {
    snprintf(msg, sizeof msg,
             "layer of %lld x %lld elements exceeds the %d elements the built-in scratch "
             "serves; use intlora_gen_aux with a workspace",
             static_cast<long long>(d), static_cast<long long>(n), INTLORA_NOALLOC_MAX_ELEMENTS);
    intlora::set_last_error(msg);
    return INTLORA_ERR_UNSUPPORTED;
  }
  intlora_aux_job job = {W,        d,           n,           seed,       stream_id,
                         alpha,    w_bits,      sigma_w_out, sigma_r_out, r_star_out,
                         w_round_out, ld_w_out, s_out,       z_out};
  if (intlora_gen_aux_workspace_size(&job, 1) > kScratchBytes) {
    intlora::set_last_error("layer needs more scratch than the built-in array holds");
    return INTLORA_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof msg, "device address of the built-in scratch: %s", cudaGetErrorString(e));
    intlora::set_last_error(msg);
    return INTLORA_ERR_CUDA;
  }
  return intlora_gen_aux(W, d, n, seed, stream_id, alpha, w_bits, sigma_w_out, sigma_r_out,
                         r_star_out, w_round_out, ld_w_out, s_out, z_out, scratch, kScratchBytes,
                         stream);
}
