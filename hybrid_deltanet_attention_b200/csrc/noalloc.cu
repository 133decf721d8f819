// A decode step whose scratch memory lives in a fixed device array of this library, for
// callers that cannot allocate device memory at the point where they step the model:
// hard real-time loops that must not hit the implicit synchronisation of cudaMalloc /
// cudaFree, and hosts that own a fixed device-memory budget and hand this library only
// the model's own buffers. It is called from ordinary host code like every other entry
// point (not from a CUDA host callback or a stream-ordered host function: CUDA allows no
// CUDA call at all there, and this function makes several).
//
// CUDA loads this library's device code lazily by default (since CUDA 12.2), so the
// scratch array is loaded and reserved on a device at the first call there (the address
// lookup below), and kept until the process exits. Every call shares it and it keeps the
// last call's contents, so calls whose kernels overlap on the GPU (on different streams,
// or from different threads) race on it; the call clears, on its stream, the part that
// must start at zero.
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "mk_model.h"

namespace {

// 4 MiB. The per-step scratch does not depend on the context length (the attention
// partials are sized by the grid and the KV heads): about 0.7 MB for the 0.8B-shaped model
// and 1.3 MB for the 27B-shaped one.
constexpr size_t kStaticScratchBytes = 4u << 20;
constexpr size_t kZeroHeadBytes = 4096;   // barrier/arrival/argmax words and per-head sums of squares
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

int fail(int code, const std::string& msg) {
  mk_set_last_error(msg);
  return code;
}

}  // namespace

extern "C" {

int mk_decode_step_noalloc(mk_model* m, const int32_t* d_in_token, int32_t* d_out_token, float* d_logits,
                           void* stream) {
  if (!m) return fail(MK_ERR_ARG, "model is NULL");
  if (!d_in_token || !d_out_token) return fail(MK_ERR_ARG, "token pointer is NULL");
  if (m->pos_hint + 1 > m->cfg.max_ctx) return fail(MK_ERR_CAPACITY, "context capacity reached");
  if (m->step_scratch_bytes > kStaticScratchBytes)
    return fail(MK_ERR_CAPACITY, "this model needs " + std::to_string(m->step_scratch_bytes) +
                                     " bytes of step scratch; the static area holds " +
                                     std::to_string(kStaticScratchBytes));
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(MK_ERR_ARG, "device index out of range");
  if (dev != m->device) return fail(MK_ERR_ARG, "the current device is not the model's device");
  void* base = nullptr;
  {
    // Once per device, with that device current: the device address of the array (in
    // host code the array's name is only a stand-in, not a device address).
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_scratch);
      if (e != cudaSuccess || !ptr)
        return fail(MK_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_scratch_addr[dev] = ptr;
    }
    base = g_scratch_addr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The sync words and the first layer's norm sums must start at zero; everything else
  // in the scratch is written before it is read within a step.
  e = cudaMemsetAsync(base, 0, kZeroHeadBytes, s);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, std::string("clearing the static scratch: ") + cudaGetErrorString(e));

  mk::DecodeParams p = m->base;
  auto rebase = [&](auto* ptr) {
    using T = decltype(ptr);
    return reinterpret_cast<T>(static_cast<unsigned char*>(base) +
                               (reinterpret_cast<const uint8_t*>(ptr) - m->ws));
  };
  p.bar = rebase(p.bar);
  p.done = rebase(p.done);
  p.amax = rebase(p.amax);
  p.ssq = rebase(p.ssq);
  p.hbuf = rebase(p.hbuf);
  p.z = rebase(p.z);
  p.ybuf = rebase(p.ybuf);
  p.part = rebase(p.part);
  p.obuf = rebase(p.obuf);
  p.abuf = rebase(p.abuf);

  p.in_token = d_in_token;
  p.out_token = d_out_token;
  p.logits = d_logits;
  e = mk::launch_decode(p, m->grid, s);
  if (e == cudaErrorCooperativeLaunchTooLarge)
    return fail(MK_ERR_RESIDENCY, std::string("persistent grid cannot be co-resident: ") + cudaGetErrorString(e));
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
  ++m->launches;
  ++m->pos_hint;
  ++m->pos_max;
  return MK_OK;
}

}  // extern "C"
