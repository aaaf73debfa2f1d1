// Internal declarations shared by the libtq translation units (host side).
#pragma once
#include <cstddef>
#include <cstdint>
#include <string>

#include "../../include/tq.h"

namespace tq {

// thread-local last-error message
tq_status fail(tq_status code, const std::string& msg);
void clear_error();

// CUDA error -> TQ_ERR_CUDA with the runtime's message
tq_status cuda_fail(int err, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---- prepared-rotation buffer layout -------------------------------------------------------------
// All regions 256-byte aligned. fp32 matrices row-major d x d; fp16 matrices row-major, padded to
// Dp x Dp (Dp = d rounded up to a multiple of 128) with zeros so tensor-core tiles never read past
// a region.
//   Pi32, S32, T32 = S Pi^T
//   Pi_hi, Pi_lo   : fp16 split of Pi       (Pi  = Pi_hi + 2^-12 Pi_lo)
//   T_hi,  T_lo    : fp16 split of T
//   PiT_hi, PiT_lo : fp16 split of Pi^T
//   ST_hi,  ST_lo  : fp16 split of S^T
struct RotLayout {
  int d, dp;
  size_t pi32, s32, t32;
  size_t pi_hi, pi_lo, t_hi, t_lo, pit_hi, pit_lo, st_hi, st_lo;
  size_t total;
};
RotLayout rot_layout(int d);

constexpr float kSplitScale = 4096.0f;      // 2^12: scale of the low fp16 part of a split
constexpr float kSplitScaleInv = 1.0f / 4096.0f;

bool valid_dim(int d);       // multiple of 32 in [32, 4096]

// Device address of the library's error word (kernels record bounded-wait timeouts there).
uint32_t* device_error_word();

// Number of SMs of the current device.
int sm_count();

}  // namespace tq
