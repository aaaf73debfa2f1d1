// tq_attend_decode_noalloc: decode attention with its scratch in a fixed, library-owned device
// array instead of a caller workspace.
//
// Who needs this: callers that cannot hand the library a device buffer. A plain C host that only
// holds the cache and query pointers has no device allocator of its own; a serving runtime that
// reserved all of HBM for its own pool up front cannot get more from cudaMalloc; and a caller on
// a latency-critical stream cannot afford cudaFree, which waits for the whole device. For them
// this entry point allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
//
// The scratch is one file-scope __device__ array per device (each device that uses the library
// holds its own copy). Its device address is looked up on every call, with the caller's device
// current: a cached address would go stale if the device's context were torn down and created
// again (the module, and with it the array, may then load elsewhere). The lookup is a host-side
// table read of the loaded module, cheap next to the launches. The array is
// shared by every call on that device, so calls whose GPU work overlaps (two streams, two host
// threads) race on it: callers must order such calls themselves (one stream, or events).
// Nothing in the array has to start at zero or survive between calls: every byte the attention
// kernels read from their scratch is written earlier in the same call.
#include <cuda_runtime.h>

#include <string>

#include "tq_internal.h"

namespace {

__device__ __align__(256) uint8_t g_attend_scratch[TQ_ATTEND_NOALLOC_MAX_BYTES];

// Device address of the current device's scratch array.
tq_status scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_attend_scratch);
  if (e != cudaSuccess || p == nullptr)
    return tq::cuda_fail(e != cudaSuccess ? (int)e : (int)cudaErrorInvalidSymbol,
                         "tq_attend_decode_noalloc: scratch address");
  *out = p;
  return TQ_OK;
}

}  // namespace

extern "C" TQ_API tq_status tq_attend_decode_noalloc(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B,
                                                     int32_t Hq, int32_t Hkv, int64_t T, int32_t d, const void* q,
                                                     int32_t q_dtype, const void* rot, const uint32_t* k_codes,
                                                     const uint16_t* k_norms, const uint32_t* k_signs,
                                                     const uint16_t* k_gammas, const uint32_t* v_codes,
                                                     const uint32_t* v_signs, const uint16_t* v_norms,
                                                     const uint16_t* v_gammas, float scale, float* out,
                                                     void* stream) {
  tq::clear_error();
  const size_t need = tq_attend_workspace_bytes(B, Hq, Hkv, T, d);
  if (need > (size_t)TQ_ATTEND_NOALLOC_MAX_BYTES)
    return tq::fail(TQ_ERR_WORKSPACE,
                    "tq_attend_decode_noalloc: these sizes need " + std::to_string(need) +
                        " bytes of scratch, more than the fixed " + std::to_string(TQ_ATTEND_NOALLOC_MAX_BYTES) +
                        "-byte array; call tq_attend_decode with a workspace instead");
  void* scratch = nullptr;
  const tq_status s = scratch_address(&scratch);
  if (s != TQ_OK) return s;
  // sizes too small to be valid (need == 0) are reported by tq_attend_decode's own checks
  return tq_attend_decode(cb_k, cb_v, B, Hq, Hkv, T, d, q, q_dtype, rot, k_codes, k_norms, k_signs, k_gammas,
                          v_codes, v_signs, v_norms, v_gammas, scale, out, scratch,
                          (size_t)TQ_ATTEND_NOALLOC_MAX_BYTES, stream);
}
