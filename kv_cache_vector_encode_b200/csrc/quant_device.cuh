// Device helpers shared by the encode kernels: the symmetric-codebook quantiser and exact
// power-of-two scaling.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace tq {

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// m = #{positive boundaries < a} by binary search over the H-1 positive boundaries.
template <int BITS>
__device__ __forceinline__ int sym_m(float a, const float (&P)[8]) {
  if (BITS == 1) return 0;
  if (BITS == 2) return a > P[0] ? 1 : 0;
  if (BITS == 3) {
    const int m1 = a > P[1] ? 1 : 0;
    const int m0 = a > (m1 ? P[2] : P[0]) ? 1 : 0;
    return 2 * m1 + m0;
  }
  const int m2 = a > P[3] ? 1 : 0;
  const int m1 = a > (m2 ? P[5] : P[1]) ? 1 : 0;
  const float p0 = m2 ? (m1 ? P[6] : P[4]) : (m1 ? P[2] : P[0]);
  const int m0 = a > p0 ? 1 : 0;
  return 4 * m2 + 2 * m1 + m0;
}

// sym_m for a width known only at run time (warp-uniform where it is used)
__device__ __forceinline__ int sym_m_rt(float a, const float (&P)[8], int bits) {
  switch (bits) {
    case 1: return sym_m<1>(a, P);
    case 2: return sym_m<2>(a, P);
    case 3: return sym_m<3>(a, P);
    default: return sym_m<4>(a, P);
  }
}

template <int BITS>
__device__ __forceinline__ float sym_c(int m, const float (&C)[8]) {
  if (BITS == 1) return C[0];
  if (BITS == 2) return m ? C[1] : C[0];
  if (BITS == 3) return (m & 2) ? ((m & 1) ? C[3] : C[2]) : ((m & 1) ? C[1] : C[0]);
  const float lo = (m & 2) ? ((m & 1) ? C[3] : C[2]) : ((m & 1) ? C[1] : C[0]);
  const float hi = (m & 2) ? ((m & 1) ? C[7] : C[6]) : ((m & 1) ? C[5] : C[4]);
  return (m & 4) ? hi : lo;
}

// two exact power-of-two factors whose product is 2^e (e may exceed the fp32 exponent range)
__device__ __forceinline__ void pow2_pair(int e, float& f1, float& f2) {
  const int e1 = max(min(e, 120), -120);
  f1 = __int_as_float((127 + e1) << 23);
  f2 = __int_as_float((127 + (e - e1)) << 23);
}

}  // namespace tq
