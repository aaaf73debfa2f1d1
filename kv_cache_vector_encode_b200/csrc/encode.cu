// Fused TurboQuant encode for d <= 128: Algorithm 1 (tq_encode_mse) and Algorithm 2
// (tq_encode_prod) in one persistent, warp-specialised tcgen05 kernel.
//
// Method (ai-navigate-news page, "how it works (technical)"; aiboss88 page, "technical
// principles"): y = Pi x / |x|, idx_j = #{k : t_k < y_j} against the Lloyd-Max boundaries, bit
// planes of idx, fp16 |x|; Algorithm 2 adds the residual rho = y - c[idx] (rotated domain; its
// norm equals |x/|x| - Pi^T c[idx]| for orthogonal Pi), gamma = |rho| and the signs of
// S r = S Pi^T rho = T rho.
//
// Orientation: the products are computed transposed, D[i][v] = sum_k A[i][k] B[v][k] with
// A = Pi (rows = output coordinates i, M = 128, zero-padded past d) resident in shared memory for
// the whole kernel and B = a tile of NV input vectors. TMEM lane i then holds coordinate i of every
// vector of the tile, so the 32 lanes of an epilogue warp are the 32 coordinates of one packing
// group and each bit plane word is a single __ballot_sync.
//
// Precision: x is scaled per vector by a power of two so |x| lies in [2^14, 2^15) and converted to
// fp16 (exact for bf16 input; fp32 input is split hi + 2^-12 lo). Pi = Pi_hi + 2^-12 Pi_lo. The
// products are exact in the tensor core and accumulate in fp32 in TMEM:
//   D_hi = Pi_hi x_hi,  D_lo = Pi_lo x_hi (+ Pi_hi x_lo),   y = (D_hi + 2^-12 D_lo) / (|x| 2^e).
// The QJL projection uses rho scaled by 2^14 and split the same way, with three products
// (T_hi rho_hi, T_lo rho_hi, T_hi rho_lo). Relative error about 2^-22, far inside the 1e-5 band.
//
// Roles (10 warps): warp 0 issues bulk copies of raw input tiles (TMA engine); warp 1 owns TMEM
// and one lane issues every MMA; warps 2-5 convert a raw tile into the fp16 B operand and compute
// the norms; warps 6-9 are the epilogue (TMEM -> quantise -> ballot -> store). Buffers: raw input
// x2, B operand x1, TMEM accumulators x2. All waits are bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kEncThreads = 320;
constexpr float kRhoScale = 16384.0f;   // 2^14: |rho| < 2 keeps rho * 2^14 below the fp16 maximum

struct EncodeParams {
  const void* x;
  int64_t n;
  int d, G, bits, L, KP, ntiles;
  const __half* pi_hi;
  const __half* pi_lo;
  const __half* t_hi;
  const __half* t_lo;
  int dp;
  uint32_t* codes;
  uint32_t* signs;
  uint16_t* norms;
  uint16_t* gammas;
  float thr[16];
  float cent[16];
  uint32_t* err;
};

struct EncLayout {
  uint32_t a_bytes, raw_bytes, bx_bytes;
  uint32_t off_a[4], off_raw[2], off_bx[2], off_rho[2];
  uint32_t off_codes, off_signs, off_info, off_gpart, off_lut, off_bar;
  uint32_t total;
};

__host__ __device__ inline uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <int ES, bool ALG2, bool SPLITX>
__host__ __device__ inline EncLayout enc_layout(int d, int KP, int NV, int G, int bits) {
  EncLayout L{};
  L.a_bytes = 128u * KP * 2;
  L.raw_bytes = round_up((uint32_t)NV * d * ES, 1024);
  L.bx_bytes = (uint32_t)NV * KP * 2;
  uint32_t off = 0;
  int na = ALG2 ? 4 : 2;
  for (int i = 0; i < na; ++i) { L.off_a[i] = off; off += L.a_bytes; }
  for (int i = 0; i < 2; ++i) { L.off_raw[i] = off; off += L.raw_bytes; }
  for (int i = 0; i < (SPLITX ? 2 : 1); ++i) { L.off_bx[i] = off; off += L.bx_bytes; }
  if (ALG2)
    for (int i = 0; i < 2; ++i) { L.off_rho[i] = off; off += L.bx_bytes; }
  L.off_codes = off; off += round_up((uint32_t)NV * G * bits * 4, 128);
  L.off_signs = off; off += round_up((uint32_t)NV * G * 4, 128);
  L.off_info = off; off += 2u * NV * 4;
  L.off_gpart = off; off += 4u * NV * 4;
  L.off_lut = off; off += 16 * 4;
  L.off_bar = round_up(off, 8); off = L.off_bar + 32 * 8;
  L.total = off + 1024;  // slack for 1024-byte alignment of the dynamic buffer
  return L;
}

enum Bars {
  RAW_FULL = 0, RAW_EMPTY = 2, BX_FULL = 4, BX_EMPTY = 5, ACC_FULL = 6, ACC_EMPTY = 8, INFO_EMPTY = 10,
  RHO_FULL = 12, T_FULL = 13, EPI = 15, NBARS = 16
};

__device__ __forceinline__ float transpose_reduce32(float (&r)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < s; ++j) {
      float send = upper ? r[j] : r[j + s];
      float keep = upper ? r[j + s] : r[j];
      r[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return r[0];
}

__device__ __forceinline__ float load_x(const uint8_t* row, int k, int ES) {
  if (ES == 2) {
    uint32_t b = *(const uint16_t*)(row + 2 * k);
    return __uint_as_float(b << 16);
  }
  return *(const float*)(row + 4 * k);
}

template <int XT, bool ALG2, int NV>
__global__ void __launch_bounds__(kEncThreads, 1) encode_kernel(const __grid_constant__ EncodeParams p) {
  constexpr int ES = XT == TQ_BF16 ? 2 : 4;
  constexpr bool SPLITX = XT == TQ_F32;
  constexpr uint32_t COLS = ALG2 ? 4 * NV : 2 * NV;       // TMEM columns per accumulator buffer
  constexpr uint32_t NCOLS = 2 * COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const EncLayout Lo = enc_layout<ES, ALG2, SPLITX>(p.d, p.KP, NV, p.G, p.bits);
  uint64_t* bar = (uint64_t*)(smem + Lo.off_bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + NBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + NBARS) + 1;
  float* info = (float*)(smem + Lo.off_info);
  float* gpart = (float*)(smem + Lo.off_gpart);
  float* lut = (float*)(smem + Lo.off_lut);
  uint32_t* codes_stage = (uint32_t*)(smem + Lo.off_codes);
  uint32_t* signs_stage = (uint32_t*)(smem + Lo.off_signs);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = p.d, KP = p.KP, G = p.G, bits = p.bits;

  // ---- set-up: resident A operands, barriers, TMEM --------------------------------------------
  {
    const __half* srcs[4] = {p.pi_hi, p.pi_lo, p.t_hi, p.t_lo};
    const int na = ALG2 ? 4 : 2;
    const int chunks = KP / 8;   // 16-byte chunks per row
    for (int m = 0; m < na; ++m) {
      uint8_t* dst = smem + Lo.off_a[m];
      for (int c = tid; c < 128 * chunks; c += kEncThreads) {
        int r = c / chunks, kc = c % chunks;
        uint4 v = *(const uint4*)(srcs[m] + (size_t)r * p.dp + kc * 8);
        *(uint4*)(dst + sw128_offset(r, kc * 16, 128)) = v;
      }
    }
    if (tid < 16) lut[tid] = p.cent[tid];
    if (tid == 0) {
      mbar_init(&bar[RAW_FULL], 1); mbar_init(&bar[RAW_FULL + 1], 1);
      mbar_init(&bar[RAW_EMPTY], 128); mbar_init(&bar[RAW_EMPTY + 1], 128);
      mbar_init(&bar[BX_FULL], 128); mbar_init(&bar[BX_EMPTY], 1);
      mbar_init(&bar[ACC_FULL], 1); mbar_init(&bar[ACC_FULL + 1], 1);
      mbar_init(&bar[ACC_EMPTY], 128); mbar_init(&bar[ACC_EMPTY + 1], 128);
      mbar_init(&bar[INFO_EMPTY], 128); mbar_init(&bar[INFO_EMPTY + 1], 128);
      mbar_init(&bar[RHO_FULL], 128);
      mbar_init(&bar[T_FULL], 1); mbar_init(&bar[T_FULL + 1], 1);
      mbar_init(&bar[EPI], 128);
      *abort_flag = 0;
      fence_mbar_init();
    }
    fence_proxy_async_smem();
    if (warp == 1) {
      tmem_alloc(tmem_slot, NCOLS);
      tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  const uint32_t tbase = *tmem_slot;
  const int my_tiles = p.ntiles > (int)blockIdx.x ? (p.ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp == 0) {
    // ---------------- producer: raw tiles through the bulk-copy engine ---------------------------
    if (lane == 0) {
      const uint8_t* xb = (const uint8_t*)p.x;
      for (int k = 0; k < my_tiles; ++k) {
        const int s = k & 1;
        const int64_t t = blockIdx.x + (int64_t)k * gridDim.x;
        if (!mbar_wait(&bar[RAW_EMPTY + s], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        const int64_t v0 = t * NV;
        const int rows = (int)min((int64_t)NV, p.n - v0);
        const uint32_t bytes = (uint32_t)rows * d * ES;
        mbar_arrive_expect_tx(&bar[RAW_FULL + s], bytes);
        bulk_g2s(smem + Lo.off_raw[s], xb + v0 * d * ES, bytes, &bar[RAW_FULL + s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ---------------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, NV);
      const uint32_t a0 = smem_u32(smem + Lo.off_a[0]), a1 = smem_u32(smem + Lo.off_a[1]);
      const uint32_t a2 = ALG2 ? smem_u32(smem + Lo.off_a[2]) : 0u, a3 = ALG2 ? smem_u32(smem + Lo.off_a[3]) : 0u;
      const uint32_t bx0 = smem_u32(smem + Lo.off_bx[0]), bx1 = SPLITX ? smem_u32(smem + Lo.off_bx[1]) : 0u;
      const uint32_t r0 = ALG2 ? smem_u32(smem + Lo.off_rho[0]) : 0u, r1 = ALG2 ? smem_u32(smem + Lo.off_rho[1]) : 0u;
      const int ksteps = KP / 16;
      auto issue_T = [&](int j) -> bool {
        const int a = j & 1;
        if (!mbar_wait(&bar[RHO_FULL], j & 1, p.err, kDevTimeoutSync, abort_flag)) return false;
        tc_fence_after();
        const uint32_t dT1 = tbase + a * COLS + 2 * NV, dT2 = dT1 + NV;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t kb = ks * 32, blk = kb >> 7, inb = kb & 127;
          const uint32_t ao = blk * 128 * 128 + inb, bo = blk * NV * 128 + inb;
          mma_f16_ss(dT1, desc_kmajor_sw128(a2 + ao), desc_kmajor_sw128(r0 + bo), idesc, ks > 0);
          mma_f16_ss(dT2, desc_kmajor_sw128(a3 + ao), desc_kmajor_sw128(r0 + bo), idesc, ks > 0);
          mma_f16_ss(dT2, desc_kmajor_sw128(a2 + ao), desc_kmajor_sw128(r1 + bo), idesc, 1);
        }
        mma_commit(&bar[T_FULL + a]);
        return true;
      };
      bool ok = true;
      for (int k = 0; k < my_tiles && ok; ++k) {
        const int a = k & 1;
        if (!mbar_wait(&bar[ACC_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        if (!mbar_wait(&bar[BX_FULL], k & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        tc_fence_after();
        const uint32_t dhi = tbase + a * COLS, dlo = dhi + NV;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t kb = ks * 32, blk = kb >> 7, inb = kb & 127;
          const uint32_t ao = blk * 128 * 128 + inb, bo = blk * NV * 128 + inb;
          const uint64_t db = desc_kmajor_sw128(bx0 + bo);
          mma_f16_ss(dhi, desc_kmajor_sw128(a0 + ao), db, idesc, ks > 0);
          mma_f16_ss(dlo, desc_kmajor_sw128(a1 + ao), db, idesc, ks > 0);
          if (SPLITX) mma_f16_ss(dlo, desc_kmajor_sw128(a0 + ao), desc_kmajor_sw128(bx1 + bo), idesc, 1);
        }
        mma_commit(&bar[BX_EMPTY]);
        mma_commit(&bar[ACC_FULL + a]);
        if (ALG2 && k >= 1) ok = issue_T(k - 1);
      }
      if (ALG2 && ok && my_tiles >= 1 && !*abort_flag) issue_T(my_tiles - 1);
    }
  } else if (warp < 6) {
    // ---------------- converters: norm, power-of-two scale, fp16 B operand ----------------------
    const int cw = warp - 2;
    const int EPL = d / 32;
    for (int k = 0; k < my_tiles; ++k) {
      const int s = k & 1, a = k & 1;
      const int64_t t = blockIdx.x + (int64_t)k * gridDim.x;
      const int64_t v0 = t * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
      if (!mbar_wait(&bar[RAW_FULL + s], (k >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag)) break;
      if (!mbar_wait(&bar[BX_EMPTY], (k & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      if (!mbar_wait(&bar[INFO_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      uint8_t* bx = smem + Lo.off_bx[0];
      uint8_t* bxl = smem + Lo.off_bx[SPLITX ? 1 : 0];
      const uint8_t* raw = smem + Lo.off_raw[s];
      for (int v = cw; v < NV; v += 4) {
        if (v < rows) {
          const uint8_t* row = raw + (size_t)v * d * ES;
          float xv[4];
          double ss = 0.0;       // fp64: squares of any bf16 / fp32 value neither overflow nor underflow
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xv[e] = 0.0f;
            if (e < EPL) {
              xv[e] = load_x(row, lane * EPL + e, ES);
              ss = fma((double)xv[e], (double)xv[e], ss);
            }
          }
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          const double nrm = sqrt(ss);
          double scale = 1.0;
          float inv = 0.0f;
          if (nrm > 0.0) {
            int E;
            frexp(nrm, &E);
            scale = ldexp(1.0, 15 - E);            // |x| * scale in [2^14, 2^15)
            inv = (float)(1.0 / (nrm * scale));
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (e < EPL) {
              const int kk = lane * EPL + e;
              const float xs = (float)((double)xv[e] * scale);
              const __half h = __float2half_rn(xs);
              *(__half*)(bx + sw128_offset(v, 2 * kk, NV)) = h;
              if (SPLITX) {
                const __half l = __float2half_rn((xs - __half2float(h)) * kSplitScale);
                *(__half*)(bxl + sw128_offset(v, 2 * kk, NV)) = l;
              }
            }
          }
          if (lane == 0) {
            info[a * NV + v] = inv;
            p.norms[v0 + v] = __half_as_ushort(__double2half(nrm));
          }
        } else {
          for (int kk = lane; kk < d; kk += 32) {
            *(__half*)(bx + sw128_offset(v, 2 * kk, NV)) = __float2half_rn(0.0f);
            if (SPLITX) *(__half*)(bxl + sw128_offset(v, 2 * kk, NV)) = __float2half_rn(0.0f);
          }
          if (lane == 0) info[a * NV + v] = 0.0f;
        }
        for (int kk = d + lane; kk < KP; kk += 32) {   // K padding
          *(__half*)(bx + sw128_offset(v, 2 * kk, NV)) = __float2half_rn(0.0f);
          if (SPLITX) *(__half*)(bxl + sw128_offset(v, 2 * kk, NV)) = __float2half_rn(0.0f);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar[RAW_EMPTY + s]);
      mbar_arrive(&bar[BX_FULL]);
    }
  } else {
    // ---------------- epilogue: quantise, ballot-pack, residual, signs -------------------------
    const int q = warp & 3;             // TMEM lane quarter = packing group
    const int i = q * 32 + lane;        // coordinate
    const bool active = i < d;
    const int te = tid - 6 * 32;        // 0..127
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    float thr[15];
#pragma unroll
    for (int kq = 0; kq < 15; ++kq) thr[kq] = p.thr[kq];
    const int nthr = p.L - 1;
    uint32_t epi_uses = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&bar[EPI]);
      bool ok = mbar_wait(&bar[EPI], epi_uses & 1, p.err, kDevTimeoutSync, abort_flag);
      ++epi_uses;
      return ok;
    };
    uint8_t* rho_hi = ALG2 ? smem + Lo.off_rho[0] : nullptr;
    uint8_t* rho_lo = ALG2 ? smem + Lo.off_rho[1] : nullptr;
    for (int k = 0; k < my_tiles; ++k) {
      const int a = k & 1;
      const int64_t t = blockIdx.x + (int64_t)k * gridDim.x;
      const int64_t v0 = t * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
      if (!mbar_wait(&bar[ACC_FULL + a], (k >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      const uint32_t dhi = tbase + lane_base + a * COLS, dlo = dhi + NV;
      for (int c0 = 0; c0 < NV; c0 += 32) {
        uint32_t hi[32], lo[32];
        tmem_ld16(dhi + c0, *(uint32_t(*)[16]) & hi[0]);
        tmem_ld16(dhi + c0 + 16, *(uint32_t(*)[16]) & hi[16]);
        tmem_ld16(dlo + c0, *(uint32_t(*)[16]) & lo[0]);
        tmem_ld16(dlo + c0 + 16, *(uint32_t(*)[16]) & lo[16]);
        tmem_ld_wait();
        uint32_t myw[4] = {0u, 0u, 0u, 0u};
        float r2[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int v = c0 + j;
          const float inv = info[a * NV + v];
          const float y = fmaf(__uint_as_float(lo[j]), kSplitScaleInv, __uint_as_float(hi[j])) * inv;
          int idx = 0;
#pragma unroll
          for (int kq = 0; kq < 15; ++kq)
            if (kq < nthr) idx += (y > thr[kq]) ? 1 : 0;
#pragma unroll
          for (int pl = 0; pl < 4; ++pl) {
            if (pl < bits) {
              const uint32_t w = __ballot_sync(0xffffffffu, active && ((idx >> pl) & 1));
              if (lane == j) myw[pl] = w;
            }
          }
          if (ALG2) {
            float rho = (active && inv != 0.0f) ? (y - lut[idx]) : 0.0f;
            r2[j] = rho * rho;
            const float rs = rho * kRhoScale;
            const __half rh = __float2half_rn(rs);
            const __half rl = __float2half_rn((rs - __half2float(rh)) * kSplitScale);
            if (i < KP) {
              const uint32_t off = sw128_offset(v, 2 * i, NV);
              *(__half*)(rho_hi + off) = rh;
              *(__half*)(rho_lo + off) = rl;
            }
          }
        }
        if (q < G) {
#pragma unroll
          for (int pl = 0; pl < 4; ++pl)
            if (pl < bits) codes_stage[((c0 + lane) * G + q) * bits + pl] = myw[pl];
        }
        if (ALG2) {
          const float tot = transpose_reduce32(r2, lane);
          gpart[q * NV + c0 + lane] = tot;
        }
      }
      if (ALG2) {
        fence_proxy_async_smem();
        mbar_arrive(&bar[RHO_FULL]);
      }
      if (!epi_sync()) break;
      {
        uint32_t* dst = p.codes + v0 * G * bits;
        const int nw = rows * G * bits;
        for (int w = te; w < nw; w += 128) dst[w] = codes_stage[w];
      }
      if (ALG2) {
        if (te < rows) {
          float g2 = 0.0f;
          for (int qq = 0; qq < G; ++qq) g2 += gpart[qq * NV + te];
          p.gammas[v0 + te] = __half_as_ushort(__float2half_rn(sqrtf(g2)));
        }
        if (!mbar_wait(&bar[T_FULL + a], (k >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
        tc_fence_after();
        const uint32_t dT1 = tbase + lane_base + a * COLS + 2 * NV, dT2 = dT1 + NV;
        for (int c0 = 0; c0 < NV; c0 += 32) {
          uint32_t s1[32], s2[32];
          tmem_ld16(dT1 + c0, *(uint32_t(*)[16]) & s1[0]);
          tmem_ld16(dT1 + c0 + 16, *(uint32_t(*)[16]) & s1[16]);
          tmem_ld16(dT2 + c0, *(uint32_t(*)[16]) & s2[0]);
          tmem_ld16(dT2 + c0 + 16, *(uint32_t(*)[16]) & s2[16]);
          tmem_ld_wait();
          uint32_t mys = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float sv = fmaf(__uint_as_float(s2[j]), kSplitScaleInv, __uint_as_float(s1[j]));
            const uint32_t w = __ballot_sync(0xffffffffu, active && sv >= 0.0f);
            if (lane == j) mys = w;
          }
          if (q < G) signs_stage[(c0 + lane) * G + q] = mys;
        }
        if (!epi_sync()) break;
        uint32_t* dst = p.signs + v0 * G;
        const int nw = rows * G;
        for (int w = te; w < nw; w += 128) dst[w] = signs_stage[w];
      }
      tc_fence_before();
      mbar_arrive(&bar[ACC_EMPTY + a]);
      mbar_arrive(&bar[INFO_EMPTY + a]);
      if (!epi_sync()) break;   // stage buffers are reused by the next tile
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, NCOLS);
  }
}

template <int XT, bool ALG2, int NV>
tq_status launch_encode(EncodeParams& p, cudaStream_t st) {
  constexpr int ES = XT == TQ_BF16 ? 2 : 4;
  const EncLayout Lo = enc_layout<ES, ALG2, XT == TQ_F32>(p.d, p.KP, NV, p.G, p.bits);
  auto kern = encode_kernel<XT, ALG2, NV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "encode: shared memory attribute");
  p.ntiles = (int)((p.n + NV - 1) / NV);
  const int grid = std::min(p.ntiles, sm_count());
  kern<<<grid, kEncThreads, Lo.total, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "encode: launch");
  return TQ_OK;
}

tq_status encode_common(const char* fn, const tq_codebook* cb, int64_t n, int32_t d, const void* x, int32_t xt,
                        const void* rot, uint32_t* codes, uint32_t* signs, uint16_t* norms, uint16_t* gammas,
                        bool alg2, void* stream) {
  clear_error();
  std::string f(fn);
  if (!cb || !rot || !codes || !norms || (n > 0 && !x)) return fail(TQ_ERR_INVALID_ARG, f + ": NULL pointer");
  if (alg2 && (!signs || !gammas)) return fail(TQ_ERR_INVALID_ARG, f + ": NULL signs / gammas");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, f + ": n < 0");
  if (!valid_dim(d)) return fail(TQ_ERR_UNSUPPORTED, f + ": d must be a multiple of 32 in [32, 4096]");
  if (cb->d != d || cb->bits < 1 || cb->bits > 4 || cb->levels != (1 << cb->bits))
    return fail(TQ_ERR_INVALID_ARG, f + ": codebook does not match d / has bad bits");
  if (xt != TQ_F32 && xt != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, f + ": x_dtype must be TQ_F32 or TQ_BF16");
  if (!aligned16(x) || !aligned16(rot) || !aligned16(codes) || !aligned16(norms) ||
      (alg2 && (!aligned16(signs) || !aligned16(gammas))))
    return fail(TQ_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  if (n == 0) return TQ_OK;
  if (d > 128) return fail(TQ_ERR_UNSUPPORTED, f + ": d > 128 is not supported by this build");
  RotLayout RL = rot_layout(d);
  const char* base = (const char*)rot;
  EncodeParams p{};
  p.x = x;
  p.n = n;
  p.d = d;
  p.G = d / 32;
  p.bits = cb->bits;
  p.L = cb->levels;
  p.KP = d <= 64 ? 64 : 128;
  p.pi_hi = (const __half*)(base + RL.pi_hi);
  p.pi_lo = (const __half*)(base + RL.pi_lo);
  p.t_hi = (const __half*)(base + RL.t_hi);
  p.t_lo = (const __half*)(base + RL.t_lo);
  p.dp = RL.dp;
  p.codes = codes;
  p.signs = signs;
  p.norms = norms;
  p.gammas = gammas;
  for (int k = 0; k < 16; ++k) {
    p.cent[k] = k < cb->levels ? cb->c[k] : 0.0f;
    p.thr[k] = k < cb->levels - 1 ? cb->t[k] : 0.0f;
  }
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, f + ": no device error word (is a CUDA device present?)");
  cudaStream_t st = (cudaStream_t)stream;
  if (!alg2) {
    return xt == TQ_BF16 ? launch_encode<TQ_BF16, false, 128>(p, st) : launch_encode<TQ_F32, false, 64>(p, st);
  }
  return xt == TQ_BF16 ? launch_encode<TQ_BF16, true, 64>(p, st) : launch_encode<TQ_F32, true, 32>(p, st);
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" TQ_API tq_status tq_encode_mse(const tq_codebook* cb, int64_t n, int32_t d, const void* x, int32_t x_dtype,
                                   const void* rot, uint32_t* codes, uint16_t* norms, void* stream) {
  return encode_common("tq_encode_mse", cb, n, d, x, x_dtype, rot, codes, nullptr, norms, nullptr, false, stream);
}

extern "C" TQ_API tq_status tq_encode_prod(const tq_codebook* cb_bm1, int64_t n, int32_t d, const void* x, int32_t x_dtype,
                                    const void* rot, uint32_t* codes, uint32_t* signs, uint16_t* norms,
                                    uint16_t* gammas, void* stream) {
  return encode_common("tq_encode_prod", cb_bm1, n, d, x, x_dtype, rot, codes, signs, norms, gammas, true, stream);
}
