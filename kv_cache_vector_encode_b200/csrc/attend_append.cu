// tq_attend_append: one decode step on a packed KV cache with room to grow. The new token's key
// and value of every (batch, KV head) slice are encoded (keys Algorithm 1, values Algorithm 2, the
// ai-navigate-news page's split) into the next free slot of that slice, then the query attends over
// all filled slots, including the new one, exactly as tq_attend_decode does over a full cache.
//
// Launches: the two encoders on the B x Hkv new vectors (into workspace, contiguous), one small
// kernel that moves each encoded record into slot T_cur of its slice, and the attention kernels
// reading the cache with a slot stride of T_max. All on the caller's stream, in that order.
#include <cuda_runtime.h>

#include <string>

#include "tq_internal.h"

namespace tq {
namespace {

// One block per new vector s (slice s): copy its key record (codes, norm) and value record
// (codes, signs, norm, gamma) from the contiguous encode output into slot t of the slice.
__global__ void append_scatter_kernel(int n, int64_t t_max, int64_t t, int kw, int vw, int sw,
                                      const uint32_t* __restrict__ kc_new, const uint16_t* __restrict__ kn_new,
                                      const uint32_t* __restrict__ vc_new, const uint32_t* __restrict__ vs_new,
                                      const uint16_t* __restrict__ vn_new, const uint16_t* __restrict__ vg_new,
                                      uint32_t* __restrict__ k_codes, uint16_t* __restrict__ k_norms,
                                      uint32_t* __restrict__ v_codes, uint32_t* __restrict__ v_signs,
                                      uint16_t* __restrict__ v_norms, uint16_t* __restrict__ v_gammas) {
  const int s = blockIdx.x;
  if (s >= n) return;
  const int64_t rec = (int64_t)s * t_max + t;
  for (int i = threadIdx.x; i < kw; i += blockDim.x) k_codes[rec * kw + i] = kc_new[(int64_t)s * kw + i];
  for (int i = threadIdx.x; i < vw; i += blockDim.x) v_codes[rec * vw + i] = vc_new[(int64_t)s * vw + i];
  if (v_signs)
    for (int i = threadIdx.x; i < sw; i += blockDim.x) v_signs[rec * sw + i] = vs_new[(int64_t)s * sw + i];
  if (threadIdx.x == 0) {
    k_norms[rec] = kn_new[s];
    v_norms[rec] = vn_new[s];
    if (v_gammas) v_gammas[rec] = vg_new[s];
  }
}

size_t al256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace: [attention workspace for T_cur + 1 tokens][new key records][new value records].
struct AppendWs {
  size_t att, kc, kn, vc, vs, vn, vg, total;
};

AppendWs append_ws(int32_t B, int32_t Hq, int32_t Hkv, int64_t T_cur, int32_t d, int kb, int vb) {
  AppendWs w{};
  const size_t n = (size_t)B * Hkv, G = (size_t)d / 32;
  size_t off = 0;
  w.att = off; off += al256(tq_attend_workspace_bytes(B, Hq, Hkv, T_cur + 1, d));
  w.kc = off; off += al256(n * G * kb * 4);
  w.kn = off; off += al256(n * 2);
  w.vc = off; off += al256(n * G * vb * 4);
  w.vs = off; off += al256(n * G * 4);
  w.vn = off; off += al256(n * 2);
  w.vg = off; off += al256(n * 2);
  w.total = off;
  return w;
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" TQ_API size_t tq_attend_append_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t T_cur, int32_t d,
                                                          int32_t k_bits, int32_t v_codebook_bits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T_cur < 0 || d <= 0 || d % 32 || Hq % Hkv || k_bits < 1 || k_bits > 4 ||
      v_codebook_bits < 1 || v_codebook_bits > 4)
    return 0;
  return append_ws(B, Hq, Hkv, T_cur, d, k_bits, v_codebook_bits).total;
}

extern "C" TQ_API tq_status tq_attend_append(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                             int32_t Hkv, int64_t T_cur, int64_t T_max, int32_t d, const void* q,
                                             int32_t q_dtype, const void* k_new, const void* v_new, int32_t x_dtype,
                                             const void* rot, uint32_t* k_codes, uint16_t* k_norms,
                                             uint32_t* v_codes, uint32_t* v_signs, uint16_t* v_norms,
                                             uint16_t* v_gammas, float scale, float* out, void* ws, size_t ws_bytes,
                                             void* stream) {
  clear_error();
  const std::string f = "tq_attend_append";
  if (!cb_k || !cb_v || !q || !k_new || !v_new || !rot || !k_codes || !k_norms || !v_codes || !v_signs || !v_norms ||
      !v_gammas || !out || !ws)
    return fail(TQ_ERR_INVALID_ARG, f + ": NULL pointer (values are Algorithm 2: signs and gammas are required)");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(TQ_ERR_INVALID_ARG, f + ": bad B / Hq / Hkv");
  if (T_cur < 0 || T_max < T_cur + 1) return fail(TQ_ERR_INVALID_ARG, f + ": need 0 <= T_cur < T_max");
  if (cb_k->d != d || cb_v->d != d) return fail(TQ_ERR_INVALID_ARG, f + ": codebook d mismatch");
  // the attention's limits, checked before anything is written to the cache
  if (d != 128) return fail(TQ_ERR_UNSUPPORTED, f + ": this build supports d = 128");
  if (Hq / Hkv > 8) return fail(TQ_ERR_UNSUPPORTED, f + ": at most 8 query heads per KV head");
  if (T_cur + 1 > ((int64_t)1 << 31)) return fail(TQ_ERR_UNSUPPORTED, f + ": T too large");
  if (cb_k->bits < 1 || cb_k->bits > 3 || cb_v->bits < 1 || cb_v->bits > 2)
    return fail(TQ_ERR_UNSUPPORTED, f + ": key codebooks of 1..3 bits, value codebooks of 1..2 bits");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, f + ": q dtype");
  if (!aligned16(k_codes) || !aligned16(v_codes) || !aligned16(v_signs) || !aligned16(ws) || !aligned16(out) ||
      !aligned16(rot))
    return fail(TQ_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  const AppendWs w = append_ws(B, Hq, Hkv, T_cur, d, cb_k->bits, cb_v->bits);
  if (ws_bytes < w.total) return fail(TQ_ERR_WORKSPACE, f + ": workspace too small");
  uint8_t* base = (uint8_t*)ws;
  const int64_t n = (int64_t)B * Hkv;
  const int G = d / 32;
  tq_status st = tq_encode_mse(cb_k, n, d, k_new, x_dtype, rot, (uint32_t*)(base + w.kc), (uint16_t*)(base + w.kn),
                               stream);
  if (st != TQ_OK) return st;
  st = tq_encode_prod(cb_v, n, d, v_new, x_dtype, rot, (uint32_t*)(base + w.vc), (uint32_t*)(base + w.vs),
                      (uint16_t*)(base + w.vn), (uint16_t*)(base + w.vg), nullptr, 0, stream);
  if (st != TQ_OK) return st;
  append_scatter_kernel<<<(int)n, 32, 0, (cudaStream_t)stream>>>(
      (int)n, T_max, T_cur, G * cb_k->bits, G * cb_v->bits, G, (const uint32_t*)(base + w.kc),
      (const uint16_t*)(base + w.kn), (const uint32_t*)(base + w.vc), (const uint32_t*)(base + w.vs),
      (const uint16_t*)(base + w.vn), (const uint16_t*)(base + w.vg), k_codes, k_norms, v_codes, v_signs, v_norms,
      v_gammas);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tq_attend_append: scatter launch");
  return attend_impl("tq_attend_append", cb_k, cb_v, B, Hq, Hkv, T_cur + 1, T_max, d, q, q_dtype, rot, k_codes,
                     k_norms, nullptr, nullptr, v_codes, v_signs, v_norms, v_gammas, scale, out, base + w.att,
                     w.kc - w.att, stream);
}
