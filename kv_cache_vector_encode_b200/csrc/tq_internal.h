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
// All regions 256-byte aligned. fp32 matrices row-major d x d. fp16 matrices are padded with zeros
// to Dp x Dp (Dp = d rounded up to a multiple of 128) and stored as shared-memory images of the
// tensor-core operand layout (K-major, 128-byte swizzle): 128-row bands of rows, each band laid out
// as Dp/64 column blocks of [128 rows x 128 bytes]; element (r, c) sits at byte
//   (r / 128) * (128 * Dp * 2) + blk * 16384 + (r % 128 / 8) * 1024 + (r % 8) * 128
//     + (((2c % 128) / 16) ^ (r % 8)) * 16 + 2c % 16,     blk = 2c / 128.
// A kernel therefore loads any (band, column-block) piece with one bulk copy.
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

// Tiled encode for d > 128 (encode_tiled.cu): workspace bytes (Algorithm 2 only) and the launch.
size_t encode_tiled_ws_bytes(int64_t n, int d, bool alg2, int nsm);
tq_status encode_tiled(const tq_codebook* cb, int64_t n, int d, const void* x, int xt, const void* rot,
                       uint32_t* codes, uint32_t* signs, uint16_t* norms, uint16_t* gammas, bool alg2, void* ws,
                       size_t ws_bytes, void* stream);

// Walsh expansion of an exactly symmetric codebook (c[L-1-k] = -c[k]): for every odd subset m of
// its bit planes (increasing m), beta_m = mean over idx of c[idx] (1 - 2 parity(idx & m)), so that
// c[idx] = sum_m beta_m prod_{p in m} (1 - 2 bit_p(idx)). Returns the number of subsets (1, 2, 4
// or 8 for 1..4 bits); mask and beta must hold 8 entries.
int walsh_planes(const tq_codebook* cb, int* mask, float* beta);

// 2-D TMA tensor map (128-byte swizzle, zero fill out of range) for a row-major [rows][cols]
// matrix of esize-byte elements; `tmap` points at a 64-byte-aligned 128-byte CUtensorMap.
bool make_tmap_2d_sw128(void* tmap, const void* base, int esize, uint64_t cols, uint64_t rows, uint32_t box_cols,
                        uint32_t box_rows);


// Decode attention over the first T token slots of every (batch, KV head) slice of a packed cache
// whose slices hold tstride >= T slots (attend.cu); tq_attend_decode is the case tstride = T.
tq_status attend_impl(const char* f, const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                      int32_t Hkv, int64_t T, int64_t tstride, int32_t d, const void* q, int32_t q_dtype,
                      const void* rot, const uint32_t* k_codes, const uint16_t* k_norms, const uint32_t* k_signs,
                      const uint16_t* k_gammas, const uint32_t* v_codes, const uint32_t* v_signs,
                      const uint16_t* v_norms, const uint16_t* v_gammas, float scale, float* out, void* ws,
                      size_t ws_bytes, void* stream);

}  // namespace tq
