// Prepared rotation operands (Pi, S, T = S Pi^T and their split-fp16 forms) and the library's
// device error word.
//
// The rotation Pi and the JL matrix S are the method's random draws (aiboss88 page, technical
// principles: random rotation; ai-navigate-news page: sign(S r) for the residual); the caller draws
// them and hands them in. The tensor-core kernels need fp16 operands, so every matrix M used in a
// product is split as M = M_hi + 2^-12 M_lo with M_hi = fp16(M) and M_lo = fp16((M - M_hi) 2^12):
// together about 22 significant bits, enough for codes that are exact outside a 1e-5 band.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {

__device__ uint32_t g_device_error = 0;

RotLayout rot_layout(int d) {
  RotLayout L{};
  L.d = d;
  L.dp = (d + 127) / 128 * 128;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t off = 256;  // header
  size_t f32 = al((size_t)d * d * 4), f16 = al((size_t)L.dp * L.dp * 2);
  L.pi32 = off; off += f32;
  L.s32 = off; off += f32;
  L.t32 = off; off += f32;
  L.pi_hi = off; off += f16;
  L.pi_lo = off; off += f16;
  L.t_hi = off; off += f16;
  L.t_lo = off; off += f16;
  L.pit_hi = off; off += f16;
  L.pit_lo = off; off += f16;
  L.st_hi = off; off += f16;
  L.st_lo = off; off += f16;
  L.total = off;
  return L;
}

namespace {

// T = S Pi^T in fp64: T[i][j] = sum_k S[i][k] Pi[j][k]; one 16x16 output tile per block.
__global__ void t_matrix_kernel(const float* __restrict__ S, const float* __restrict__ Pi, float* __restrict__ T,
                                int d) {
  __shared__ double sS[16][17], sP[16][17];
  int i = blockIdx.y * 16 + threadIdx.y, j = blockIdx.x * 16 + threadIdx.x;
  double acc = 0.0;
  for (int k0 = 0; k0 < d; k0 += 16) {
    int kk = k0 + threadIdx.x;
    sS[threadIdx.y][threadIdx.x] = (i < d && kk < d) ? (double)S[(size_t)i * d + kk] : 0.0;
    int jj = blockIdx.x * 16 + threadIdx.y;
    sP[threadIdx.y][threadIdx.x] = (jj < d && kk < d) ? (double)Pi[(size_t)jj * d + kk] : 0.0;
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) acc += sS[threadIdx.y][k] * sP[threadIdx.x][k];
    __syncthreads();
  }
  if (i < d && j < d) T[(size_t)i * d + j] = (float)acc;
}

// hi/lo fp16 split of M (or of M^T when transpose), zero padded to dp x dp, written as the
// shared-memory image the tensor-core kernels use (see RotLayout): element (r, c) goes to
//   (r / 128) * (128 * dp * 2) + sw128_offset(r % 128, 2 c, 128)   bytes.
// The transposed images (read only by the decoder) hold in column c of each 32-column group the
// coordinate 16 half + 4 n + s for c % 32 = 8 s + 4 half + n: the order in which the decoder's
// byte-permute unpack produces a group.
__global__ void split_kernel(const float* __restrict__ M, int d, int dp, bool transpose, __half* __restrict__ hi,
                             __half* __restrict__ lo) {
  size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (size_t)dp * dp) return;
  int r = (int)(idx / dp), c = (int)(idx % dp);
  float v = 0.0f;
  if (transpose) {
    const int kk = c & 31;
    const int cc = (c & ~31) + 16 * ((kk >> 2) & 1) + 4 * (kk & 3) + (kk >> 3);
    if (r < d && cc < d) v = M[(size_t)cc * d + r];
  } else if (r < d && c < d) {
    v = M[(size_t)r * d + c];
  }
  __half h = __float2half_rn(v);
  __half l = __float2half_rn((v - __half2float(h)) * kSplitScale);
  size_t off = (size_t)(r >> 7) * (128u * dp * 2) + sw128_offset(r & 127, 2 * c, 128);
  hi[off / 2] = h;
  lo[off / 2] = l;
}

__global__ void header_kernel(int* hdr, int d) {
  hdr[0] = 0x54515231;  // "TQR1"
  hdr[1] = d;
}

}  // namespace

uint32_t* device_error_word() {
  static thread_local int dev = -1;
  static thread_local uint32_t* ptr = nullptr;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != dev || !ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    ptr = (uint32_t*)p;
    dev = cur;
  }
  return ptr;
}

int sm_count() {
  static thread_local int dev = -1, count = 0;
  int cur = 0;
  cudaGetDevice(&cur);
  if (cur != dev || count <= 0) {
    cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, cur);
    dev = cur;
  }
  return count > 0 ? count : 1;
}

tq_status cuda_fail(int err, const char* what) {
  return fail(TQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString((cudaError_t)err));
}

}  // namespace tq

using namespace tq;

extern "C" TQ_API size_t tq_rotation_bytes(int32_t d) {
  if (!valid_dim(d)) return 0;
  return rot_layout(d).total;
}

extern "C" TQ_API tq_status tq_rotation_prepare(int32_t d, const float* Pi, const float* S, void* rot, size_t rot_bytes,
                                         void* stream) {
  clear_error();
  if (!valid_dim(d)) return fail(TQ_ERR_UNSUPPORTED, "tq_rotation_prepare: d must be a multiple of 32 in [32, 4096]");
  if (!Pi || !S || !rot) return fail(TQ_ERR_INVALID_ARG, "tq_rotation_prepare: NULL pointer");
  if (!aligned16(Pi) || !aligned16(S) || !aligned16(rot))
    return fail(TQ_ERR_INVALID_ARG, "tq_rotation_prepare: pointers must be 16-byte aligned");
  RotLayout L = rot_layout(d);
  if (rot_bytes < L.total) return fail(TQ_ERR_WORKSPACE, "tq_rotation_prepare: rot buffer too small");
  cudaStream_t st = (cudaStream_t)stream;
  char* base = (char*)rot;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(base + L.pi32, Pi, (size_t)d * d * 4, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
    return cuda_fail(e, "tq_rotation_prepare: copy Pi");
  if ((e = cudaMemcpyAsync(base + L.s32, S, (size_t)d * d * 4, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
    return cuda_fail(e, "tq_rotation_prepare: copy S");
  dim3 tb(16, 16), tg((d + 15) / 16, (d + 15) / 16);
  t_matrix_kernel<<<tg, tb, 0, st>>>(S, Pi, (float*)(base + L.t32), d);
  size_t nel = (size_t)L.dp * L.dp;
  int blocks = (int)((nel + 255) / 256);
  split_kernel<<<blocks, 256, 0, st>>>(Pi, d, L.dp, false, (__half*)(base + L.pi_hi), (__half*)(base + L.pi_lo));
  split_kernel<<<blocks, 256, 0, st>>>((const float*)(base + L.t32), d, L.dp, false, (__half*)(base + L.t_hi),
                                       (__half*)(base + L.t_lo));
  split_kernel<<<blocks, 256, 0, st>>>(Pi, d, L.dp, true, (__half*)(base + L.pit_hi), (__half*)(base + L.pit_lo));
  split_kernel<<<blocks, 256, 0, st>>>(S, d, L.dp, true, (__half*)(base + L.st_hi), (__half*)(base + L.st_lo));
  header_kernel<<<1, 1, 0, st>>>((int*)base, d);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tq_rotation_prepare: launch");
  return TQ_OK;
}

extern "C" TQ_API tq_status tq_sync_check(void* stream) {
  clear_error();
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_sync_check");
  uint32_t v = 0, zero = 0;
  if ((e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v))) != cudaSuccess) return cuda_fail(e, "tq_sync_check");
  if (v != 0) {
    cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
    return fail(TQ_ERR_DEVICE_TIMEOUT, "a libtq kernel gave up a bounded wait (device code " + std::to_string(v) + ")");
  }
  return TQ_OK;
}
