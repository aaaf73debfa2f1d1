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
// Quantiser: the Lloyd-Max codebook is exactly symmetric (c_{L-1-k} = -c_k, t_{L/2-1} = 0), so the
// top index bit is [y > 0] and the lower bits are m XOR [y <= 0], where m counts the positive
// boundaries below |y| (a binary search of BITS-1 compares); c[idx] = +-C[m].
//
// Precision: x is scaled per vector by a power of two so |x| lies in [2^14, 2^15) and converted to
// fp16 (exact for bf16 input; fp32 input is split hi + 2^-12 lo). Pi = Pi_hi + 2^-12 Pi_lo. The
// products are exact in the tensor core and accumulate in fp32 in TMEM:
//   D_hi = Pi_hi x_hi,  D_lo = Pi_lo x_hi (+ Pi_hi x_lo),   y = (D_hi + 2^-12 D_lo) / (|x| 2^e).
// The QJL projection uses rho scaled by 2^14 and split the same way, with three products
// (T_hi rho_hi, T_lo rho_hi, T_hi rho_lo). Relative error about 2^-22, far inside the 1e-5 band.
//
// Data movement: the resident operands arrive by one bulk copy each (the prepared rotation buffer
// stores them as shared-memory images); input tiles arrive by 2-D TMA loads with 128-byte swizzle,
// i.e. already in the tensor-core operand layout, with out-of-range rows / columns zero-filled.
// bf16 tiles are converted to fp16 in place.
//
// Roles: warp 0 issues the bulk / TMA copies; warp 1 owns TMEM and issues the products of x; then
// the converters (norm, power-of-two scale, fp16; 4 warps, or 8 with two threads per vector for
// Algorithm 1 on 128-vector tiles); then 8 epilogue warps (two per TMEM lane quarter, splitting the
// vectors of a tile); and for Algorithm 2 a last warp that issues the T rho products (14 to 18 warps
// in all). Buffers: input stage x2, TMEM accumulators x2. All waits are bounded (sm100.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "quant_device.cuh"
#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

// converter warps: 8 for Algorithm 1 on 128-vector tiles (two threads per vector), else 4
__host__ __device__ constexpr int enc_conv_warps(bool alg2, int nv) { return !alg2 && nv == 128 ? 8 : 4; }
// threads: producer, MMA, converters, 8 epilogue warps, and (Algorithm 2) one that issues the T rho
// products
__host__ __device__ constexpr int enc_threads(bool alg2, int nv) {
  return 32 * (2 + enc_conv_warps(alg2, nv) + 8 + (alg2 ? 1 : 0));
}
constexpr float kRhoScale = 16384.0f;   // 2^14: |rho| < 2 keeps rho * 2^14 below the fp16 maximum

struct EncodeParams {
  int64_t n;
  int d, G, KP, ntiles;
  const uint8_t* img[4];     // Pi_hi, Pi_lo, T_hi, T_lo shared-memory images (band 0)
  uint32_t img_bytes;        // bytes of one resident operand (128 rows x KP fp16)
  uint32_t* codes;
  uint32_t* signs;
  uint16_t* norms;
  uint16_t* gammas;
  float P[8];                // positive boundaries t_{L/2} .. t_{L-2}
  float C[8];                // positive centroids c_{L/2} .. c_{L-1}
  // mixed widths per channel group (BITS == 0): group g's width, its first word in the record,
  // the record's words, and the group's positive boundaries
  int gbits[4], goff[4], wv;
  float Pm[4][8];
  uint32_t* err;
};

struct EncLayout {
  uint32_t a_bytes, raw_bytes, bx_bytes;
  uint32_t off_a[4], off_raw[2], off_bx[2][2], off_rho[2];
  uint32_t off_codes, off_signs, off_info, off_gpart, off_bar;
  uint32_t total;
};

__host__ __device__ inline uint32_t round_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }


// raw tile: bf16 -> NV rows x KP columns (KP/64 boxes of 64 columns); fp32 -> NV rows x DF columns
// (DF = d rounded up to 32, DF/32 boxes of 32 columns).
template <int XT, bool ALG2, int NV, int BITS>
__host__ __device__ inline EncLayout enc_layout(int d, int KP, int G) {
  constexpr bool F32 = XT == TQ_F32;
  EncLayout L{};
  L.a_bytes = 128u * KP * 2;
  L.raw_bytes = F32 ? (uint32_t)NV * round_up(d, 32) * 4 : (uint32_t)NV * KP * 2;
  L.bx_bytes = (uint32_t)NV * KP * 2;
  uint32_t off = 0;
  for (int i = 0; i < (ALG2 ? 4 : 2); ++i) { L.off_a[i] = off; off += L.a_bytes; }
  for (int s = 0; s < 2; ++s) { L.off_raw[s] = off; off += round_up(L.raw_bytes, 1024); }
  if (F32)
    for (int s = 0; s < 2; ++s)
      for (int h = 0; h < 2; ++h) { L.off_bx[s][h] = off; off += L.bx_bytes; }
  if (ALG2)
    for (int h = 0; h < 2; ++h) { L.off_rho[h] = off; off += L.bx_bytes; }
  // code, sign and gamma staging of the epilogue: two of each (tile parity), so that one
  // synchronisation of the epilogue warps per tile suffices
  L.off_codes = off; off += 2 * round_up((uint32_t)NV * G * BITS * 4, 128);
  L.off_signs = off; off += 2 * round_up((uint32_t)NV * G * 4, 128);
  L.off_info = off; off += 2u * NV * 4;
  L.off_gpart = off; off += 2 * 4u * NV * 4;
  L.off_bar = round_up(off, 8); off = L.off_bar + 32 * 8;
  L.total = off + 1024;  // slack for 1024-byte alignment of the dynamic buffer
  return L;
}

enum Bars {
  A_FULL = 0, RAW_FULL = 1, STAGE_EMPTY = 3, STAGE_READY = 5, ACC_FULL = 7, ACC_EMPTY = 9, INFO_EMPTY = 11,
  RHO_FULL = 13, T_FULL = 14, EPI = 16, NBARS = 17
};

// Sum over the 32 lanes of r[lane & 15] for 16 values per lane: lane l (and l ^ 16) gets the total
// for column l & 15.
__device__ __forceinline__ float transpose_reduce16(float (&r)[16], int lane) {
#pragma unroll
  for (int s = 8; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < s; ++j) {
      float send = upper ? r[j] : r[j + s];
      float keep = upper ? r[j + s] : r[j];
      r[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return r[0] + __shfl_xor_sync(0xffffffffu, r[0], 16);
}

template <int XT, bool ALG2, int NV, int BITS>
__global__ void __launch_bounds__(enc_threads(ALG2, NV), 1)
    encode_kernel(const __grid_constant__ EncodeParams p, const __grid_constant__ CUtensorMap tmap) {
  constexpr bool F32 = XT == TQ_F32;
  constexpr bool MIX = BITS == 0;                          // widths per channel group (Algorithm 1)
  constexpr int BMAX = MIX ? 4 : BITS;                     // planes of the widest group
  static_assert(!(MIX && ALG2), "mixed widths are an Algorithm 1 format");
  constexpr uint32_t COLS = ALG2 ? 4 * NV : 2 * NV;       // TMEM columns per accumulator buffer
  constexpr uint32_t NCOLS = 2 * COLS;
  constexpr int NCV = enc_conv_warps(ALG2, NV);            // converter warps (2 .. 1 + NCV)
  constexpr int TPV = 32 * NCV / NV;                       // converter threads per vector
  constexpr int W_EPI = 2 + NCV;                           // first of the 8 epilogue warps
  constexpr int W_T = W_EPI + 8;                           // T rho issuer (Algorithm 2)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int d = p.d, KP = p.KP, G = p.G;
  const EncLayout Lo = enc_layout<XT, ALG2, NV, BMAX>(d, KP, G);
  uint64_t* bar = (uint64_t*)(smem + Lo.off_bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + NBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + NBARS) + 1;
  float* info = (float*)(smem + Lo.off_info);
  float* gpart0 = (float*)(smem + Lo.off_gpart);
  uint32_t* codes_stage0 = (uint32_t*)(smem + Lo.off_codes);
  uint32_t* signs_stage0 = (uint32_t*)(smem + Lo.off_signs);
  const uint32_t codes_words = (Lo.off_signs - Lo.off_codes) / 8, signs_words = (Lo.off_info - Lo.off_signs) / 8;
  // stage-indexed buffers by arithmetic (keeps the layout struct out of local memory)
  const uint32_t raw0 = Lo.off_raw[0], raw_stride = Lo.off_raw[1] - Lo.off_raw[0];
  const uint32_t bx0 = F32 ? Lo.off_bx[0][0] : 0u, bx_stride = F32 ? Lo.off_bx[1][0] - Lo.off_bx[0][0] : 0u;
  const uint32_t bx_lo = F32 ? Lo.off_bx[0][1] - Lo.off_bx[0][0] : 0u;
  auto raw_off = [&](int s) { return raw0 + s * raw_stride; };
  auto bxh_off = [&](int s) { return bx0 + s * bx_stride; };
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bar[A_FULL], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[RAW_FULL + s], 1);
      mbar_init(&bar[STAGE_EMPTY + s], 1);
      mbar_init(&bar[STAGE_READY + s], NCV);   // one arrival per converter warp
      mbar_init(&bar[ACC_FULL + s], 1);
      mbar_init(&bar[ACC_EMPTY + s], 8);       // one arrival per epilogue warp
      mbar_init(&bar[INFO_EMPTY + s], 8);
      mbar_init(&bar[T_FULL + s], 1);
    }
    mbar_init(&bar[RHO_FULL], 8);
    mbar_init(&bar[EPI], 8);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, NCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int my_tiles = p.ntiles > (int)blockIdx.x ? (p.ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  constexpr int na = ALG2 ? 4 : 2;

  if (warp == 0) {
    // ---------------- producer: resident operands (bulk), input tiles (TMA) ----------------------
    // warp-uniform schedule; one elected lane issues the copies
    if (elect_one_sync()) {
      mbar_arrive_expect_tx(&bar[A_FULL], na * p.img_bytes);
      for (int m = 0; m < na; ++m) bulk_g2s(smem + Lo.off_a[m], p.img[m], p.img_bytes, &bar[A_FULL]);
    }
    __syncwarp();
    const int nbox = F32 ? (d + 31) / 32 : KP / 64;
    const uint32_t box_bytes = NV * 128;
    for (int k = 0; k < my_tiles; ++k) {
      const int s = k & 1;
      const int t = blockIdx.x + k * gridDim.x;
      if (!mbar_wait_warp(&bar[STAGE_EMPTY + s], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(&bar[RAW_FULL + s], nbox * box_bytes);
        for (int b = 0; b < nbox; ++b)
          tma_load_2d(smem + raw_off(s) + b * box_bytes, &tmap, b * (F32 ? 32 : 64), t * NV, &bar[RAW_FULL + s]);
      }
      __syncwarp();
    }
  } else if (warp == 1 || (ALG2 && warp == W_T)) {
    // ---------------- MMA issuers ---------------------------------------------------------------
    // warp 1 issues the products of x, warp W_T (Algorithm 2) those of rho, so that the T rho
    // products of a tile start as soon as its rho is written, not after the next tile's x products.
    // Warp-uniform schedules (descriptors stay in uniform registers); one elected lane issues.
    if (mbar_wait_warp(&bar[A_FULL], 0, p.err, kDevTimeoutLoad, abort_flag)) {
      const uint32_t idesc = idesc_f16_f32(128, NV);
      const uint32_t a0 = smem_u32(smem + Lo.off_a[0]), a1 = smem_u32(smem + Lo.off_a[1]);
      const uint32_t a2 = ALG2 ? smem_u32(smem + Lo.off_a[2]) : 0u, a3 = ALG2 ? smem_u32(smem + Lo.off_a[3]) : 0u;
      const uint32_t r0 = ALG2 ? smem_u32(smem + Lo.off_rho[0]) : 0u, r1 = ALG2 ? smem_u32(smem + Lo.off_rho[1]) : 0u;
      const int ksteps = KP / 16;
      // With NV = 64, rho is stored MN-major: one 128-byte row (the 64 vectors) per coordinate, so
      // the K = 16 slice of a step is 16 rows (2048 bytes) on. Otherwise K-major like x.
      constexpr bool RHO_MN = NV == 64;
      const uint32_t idesc_t = RHO_MN ? (idesc | (1u << 16)) : idesc;   // B (rho) MN-major
      auto issue_T = [&](int j) -> bool {
        const int a = j & 1;
        if (!mbar_wait_warp(&bar[RHO_FULL], j & 1, p.err, kDevTimeoutSync, abort_flag)) return false;
        tc_fence_after();
        const uint32_t dT1 = tbase + a * COLS + 2 * NV, dT2 = dT1 + NV;
        if (elect_one_sync()) {
          for (int ks = 0; ks < ksteps; ++ks) {
            const uint32_t kb = ks * 32, blk = kb >> 7, inb = kb & 127;
            const uint32_t ao = blk * 128 * 128 + inb;
            const uint32_t bo = RHO_MN ? ks * 16 * 128 : blk * NV * 128 + inb;
            const uint64_t d0 = RHO_MN ? desc_smem(r0 + bo, 1024, 1024, 2) : desc_kmajor_sw128(r0 + bo);
            const uint64_t d1 = RHO_MN ? desc_smem(r1 + bo, 1024, 1024, 2) : desc_kmajor_sw128(r1 + bo);
            mma_f16_ss(dT1, desc_kmajor_sw128(a2 + ao), d0, idesc_t, ks > 0);
            mma_f16_ss(dT2, desc_kmajor_sw128(a3 + ao), d0, idesc_t, ks > 0);
            mma_f16_ss(dT2, desc_kmajor_sw128(a2 + ao), d1, idesc_t, 1);
          }
          mma_commit(&bar[T_FULL + a]);
        }
        __syncwarp();
        return true;
      };
      bool ok = true;
      if (ALG2 && warp == W_T) {
        for (int j = 0; j < my_tiles && ok; ++j) ok = issue_T(j);
        ok = false;                                  // the x products are warp 1's
      }
      for (int k = 0; k < my_tiles && ok; ++k) {
        const int a = k & 1, s = k & 1;
        if (!mbar_wait_warp(&bar[ACC_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        if (!mbar_wait_warp(&bar[STAGE_READY + s], (k >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        tc_fence_after();
        const uint32_t bh = smem_u32(smem + (F32 ? bxh_off(s) : raw_off(s)));
        const uint32_t bl = F32 ? smem_u32(smem + bxh_off(s) + bx_lo) : 0u;
        const uint32_t dhi = tbase + a * COLS, dlo = dhi + NV;
        if (elect_one_sync()) {
          for (int ks = 0; ks < ksteps; ++ks) {
            const uint32_t kb = ks * 32, blk = kb >> 7, inb = kb & 127;
            const uint32_t ao = blk * 128 * 128 + inb, bo = blk * NV * 128 + inb;
            const uint64_t db = desc_kmajor_sw128(bh + bo);
            mma_f16_ss(dhi, desc_kmajor_sw128(a0 + ao), db, idesc, ks > 0);
            mma_f16_ss(dlo, desc_kmajor_sw128(a1 + ao), db, idesc, ks > 0);
            if (F32) mma_f16_ss(dlo, desc_kmajor_sw128(a0 + ao), desc_kmajor_sw128(bl + bo), idesc, 1);
          }
          mma_commit(&bar[STAGE_EMPTY + s]);
          mma_commit(&bar[ACC_FULL + a]);
        }
        __syncwarp();
      }
    }
  } else if (warp < W_EPI) {
    // ---------------- converters: one thread per vector (TPV threads when NV < 128) -------------
    const int ct = tid - 64;
    const int v = ct / TPV, part = ct % TPV;
    for (int k = 0; k < my_tiles; ++k) {
      const int s = k & 1;
      const int64_t v0 = (int64_t)(blockIdx.x + k * gridDim.x) * NV;
      if (!mbar_wait_warp(&bar[RAW_FULL + s], (k >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag)) break;
      if (!mbar_wait_warp(&bar[INFO_EMPTY + s], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      uint8_t* raw = smem + raw_off(s);
      double ss = 0.0;
      if (!F32) {
        // four independent fp64 partial sums (one per 32-bit word of a 16-byte chunk), so the
        // sum of squares is not one long chain of dependent FMAs
        const int cpp = (KP / 8) / TPV;   // 16-byte chunks (8 values) per thread
        double s4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
        for (int c = part * cpp; c < (part + 1) * cpp; ++c) {
          const uint4 w = *(const uint4*)(raw + sw128_offset(v, c * 16, NV));
          auto acc = [&](double& a, uint32_t u) {
            const double lo = __uint_as_float(u << 16), hi = __uint_as_float(u & 0xFFFF0000u);
            a = fma(lo, lo, a);
            a = fma(hi, hi, a);
          };
          acc(s4[0], w.x);
          acc(s4[1], w.y);
          acc(s4[2], w.z);
          acc(s4[3], w.w);
        }
        ss = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      } else {
        const int nch = (d + 3) / 4;            // 16-byte chunks of 4 floats actually holding data
        const int cpp = (nch + TPV - 1) / TPV;
        for (int c = part * cpp; c < min(nch, (part + 1) * cpp); ++c) {
          const float4 f = *(const float4*)(raw + sw128_offset(v, c * 16, NV));
          ss = fma((double)f.x, (double)f.x, ss);
          ss = fma((double)f.y, (double)f.y, ss);
          ss = fma((double)f.z, (double)f.z, ss);
          ss = fma((double)f.w, (double)f.w, ss);
        }
      }
#pragma unroll
      for (int o = 1; o < TPV; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const double nrm = sqrt(ss);
      float f1 = 1.0f, f2 = 1.0f, inv = 0.0f;
      if (nrm > 0.0) {
        int E;
        frexp(nrm, &E);
        pow2_pair(15 - E, f1, f2);                         // |x| * f1 * f2 in [2^14, 2^15)
        inv = (float)(1.0 / ldexp(nrm, 15 - E));
      }
      if (!F32) {
        const int cpp = (KP / 8) / TPV;
        for (int c = part * cpp; c < (part + 1) * cpp; ++c) {
          uint4* ptr = (uint4*)(raw + sw128_offset(v, c * 16, NV));
          const uint4 w = *ptr;
          auto cvt = [&](uint32_t u) -> uint32_t {
            const __half2 hh = __floats2half2_rn(__uint_as_float(u << 16) * f1 * f2,
                                                 __uint_as_float(u & 0xFFFF0000u) * f1 * f2);
            return h2_bits(hh);
          };
          *ptr = make_uint4(cvt(w.x), cvt(w.y), cvt(w.z), cvt(w.w));
        }
      } else {
        uint8_t* bxh = smem + bxh_off(s);
        uint8_t* bxl = bxh + bx_lo;
        const int nout = KP / 8;                 // 16-byte fp16 chunks of the operand row
        const int cpp = nout / TPV;
        for (int c = part * cpp; c < (part + 1) * cpp; ++c) {
          uint4 wh = make_uint4(0, 0, 0, 0), wl = wh;
          if (c * 8 < d) {
            const float4 fa = *(const float4*)(raw + sw128_offset(v, (2 * c) * 16, NV));
            const float4 fb = *(const float4*)(raw + sw128_offset(v, (2 * c + 1) * 16, NV));
            // hi = fp16(x s), lo = fp16((x s - hi) 2^12) for a pair of values
            auto split = [&](float a, float b, uint32_t& h, uint32_t& l) {
              const float x0 = a * f1 * f2, x1 = b * f1 * f2;
              const __half2 hh = __floats2half2_rn(x0, x1);
              const float2 back = __half22float2(hh);
              h = h2_bits(hh);
              l = h2_bits(__floats2half2_rn((x0 - back.x) * kSplitScale, (x1 - back.y) * kSplitScale));
            };
            split(fa.x, fa.y, wh.x, wl.x);
            split(fa.z, fa.w, wh.y, wl.y);
            split(fb.x, fb.y, wh.z, wl.z);
            split(fb.z, fb.w, wh.w, wl.w);
          }
          *(uint4*)(bxh + sw128_offset(v, c * 16, NV)) = wh;
          *(uint4*)(bxl + sw128_offset(v, c * 16, NV)) = wl;
        }
      }
      if (part == 0) {
        info[s * NV + v] = inv;
        if (v0 + v < p.n) p.norms[v0 + v] = __half_as_ushort(__double2half(nrm));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[STAGE_READY + s]);
    }
  } else if (warp < W_EPI + 8) {
    // ---------------- epilogue: quantise, ballot-pack, residual, signs -------------------------
    const int e = warp - W_EPI;             // 0..7
    const int q = warp & 3;                 // TMEM lane quarter = packing group
    const int i = q * 32 + lane;            // coordinate
    const bool active = i < d;
    const int te = tid - W_EPI * 32;        // 0..255
    const int cbeg = (e >> 2) * (NV / 2), cend = cbeg + NV / 2;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    float P[8], C[8];
    const int gq = q < G ? q : 0;
    const int gbw = MIX ? p.gbits[gq] : BITS;   // this warp's group width (warp-uniform)
    const int wrec = MIX ? p.wv : G * BITS;     // words of a vector's codes
    const int woff = MIX ? p.goff[gq] : q * BITS;
#pragma unroll
    for (int kq = 0; kq < 8; ++kq) {
      P[kq] = MIX ? p.Pm[gq][kq] : p.P[kq];
      C[kq] = p.C[kq];
    }
    uint32_t epi_uses = 0;
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[EPI]);
      bool ok = mbar_wait_warp(&bar[EPI], epi_uses & 1, p.err, kDevTimeoutSync, abort_flag);
      ++epi_uses;
      return ok;
    };
    uint8_t* rho_hi = ALG2 ? smem + Lo.off_rho[0] : nullptr;
    uint8_t* rho_lo = ALG2 ? smem + Lo.off_rho[1] : nullptr;
    // Algorithm 2 runs the epilogue one tile behind for the signs: tile k is quantised and its rho
    // kept in registers while the T rho products of tile k-1 finish; then the signs of tile k-1 are
    // read, and only then is rho of tile k stored (the rho buffer is free once those products are
    // done) and handed to the T rho issuer. One extra pass finishes the last tile's signs.
    constexpr int NB = NV / 32, NB_UNROLL = ALG2 ? NV / 32 : 1;
    int64_t v0p = 0;
    int rowsp = 0;
    for (int k = 0; k < my_tiles + (ALG2 ? 1 : 0); ++k) {
      const bool has_tile = k < my_tiles;
      const int a = k & 1;
      // this iteration's staging buffers (the other pair may still be read by slower warps)
      uint32_t* codes_stage = codes_stage0 + a * codes_words;
      uint32_t* signs_stage = signs_stage0 + a * signs_words;
      float* gpart = gpart0 + a * 4 * NV;
      const int64_t v0 = (int64_t)(blockIdx.x + k * gridDim.x) * NV;
      const int rows = has_tile ? (int)min((int64_t)NV, p.n - v0) : 0;
      uint32_t rhw[NV / 32][8], rlw[NV / 32][8];   // NV = 64: fp16 words of rho 2^14 per batch
      __half rhs[16], rls[16];                                       // NV = 32: one half per vector
      if (has_tile) {
        if (!mbar_wait_warp(&bar[ACC_FULL + a], (k >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
        tc_fence_after();
        const uint32_t dhi = tbase + lane_base + a * COLS, dlo = dhi + NV;
        // batches of 16 vectors inside this warp's half (unrolled with Algorithm 2, whose rho of
        // each batch stays in registers)
#pragma unroll NB_UNROLL
        for (int bt = 0; bt < NB; ++bt) {
          const int c0 = cbeg + 16 * bt;
          uint32_t hi[16], lo[16];
          tmem_ld16(dhi + c0, hi);
          tmem_ld16(dlo + c0, lo);
          tmem_ld_wait();
          uint32_t myw[BMAX];
#pragma unroll
          for (int pl = 0; pl < BMAX; ++pl) myw[pl] = 0u;
          float r2[16];                       // rho * 2^14 of the 16 vectors (Algorithm 2)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int v = c0 + j;
            const float inv = info[a * NV + v];
            const float y = fmaf(__uint_as_float(lo[j]), kSplitScaleInv, __uint_as_float(hi[j])) * inv;
            const bool neg = !(y > 0.0f);
            const int m = MIX ? sym_m_rt(fabsf(y), P, gbw) : sym_m<BMAX>(fabsf(y), P);
#pragma unroll
            for (int pl = 0; pl < BMAX; ++pl) {
              if (MIX && pl >= gbw) break;            // warp-uniform
              const bool bit = pl == gbw - 1 ? !neg : ((((m >> pl) & 1) != 0) != neg);
              const uint32_t w = __ballot_sync(0xffffffffu, active && bit);
              if (lane == j) myw[pl] = w;
            }
            if (ALG2) {
              const float cm = sym_c<BMAX>(m, C);
              float rho = neg ? y + cm : y - cm;
              if (!active || inv == 0.0f) rho = 0.0f;
              if (NV == 64) {
                r2[j] = rho * kRhoScale;            // packed below, two vectors per word
              } else {
                // K-major rho (32-vector tiles): one fp16 per (vector row, coordinate), kept
                r2[j] = rho * rho;
                const float rs = rho * kRhoScale;
                rhs[j] = __float2half_rn(rs);
                rls[j] = __float2half_rn((rs - __half2float(rhs[j])) * kSplitScale);
              }
            }
          }
          if (ALG2) {
            if (NV == 64) {
              // fp16 hi / lo split of rho 2^14, two vectors per word, kept for this coordinate's row
#pragma unroll
              for (int jp = 0; jp < 8; ++jp) {
                const __half2 h2 = __floats2half2_rn(r2[2 * jp], r2[2 * jp + 1]);
                const float2 back = __half22float2(h2);
                rhw[bt][jp] = h2_bits(h2);
                rlw[bt][jp] = h2_bits(__floats2half2_rn((r2[2 * jp] - back.x) * kSplitScale,
                                                                       (r2[2 * jp + 1] - back.y) * kSplitScale));
              }
              // |rho|^2 terms: (rho 2^14)^2 2^-28 rounds exactly like rho^2 (power-of-two scaling)
#pragma unroll
              for (int j = 0; j < 16; ++j) r2[j] = r2[j] * r2[j] * (1.0f / 268435456.0f);
            }
          }
          if (q < G && lane < 16) {
#pragma unroll
            for (int pl = 0; pl < BMAX; ++pl)
              if (!MIX || pl < gbw) codes_stage[(c0 + lane) * wrec + woff + pl] = myw[pl];
          }
          if (ALG2) {
            const float tot = transpose_reduce16(r2, lane);
            if (lane < 16) gpart[q * NV + c0 + lane] = tot;
          }
        }
        if (ALG2) {
          // the tile's products of x and its scales are consumed: the next-but-one tile may use them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar[ACC_EMPTY + a]);
            mbar_arrive(&bar[INFO_EMPTY + a]);
          }
        }
      }
      if (ALG2) {
        if (k >= 1) {
          // signs of tile k-1: sign(S r) = sign(T rho) from its T rho products
          const int ap = (k - 1) & 1;
          if (!mbar_wait_warp(&bar[T_FULL + ap], ((k - 1) >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
          tc_fence_after();
          const uint32_t dT1 = tbase + lane_base + ap * COLS + 2 * NV, dT2 = dT1 + NV;
          // eight vectors per TMEM load: this pass runs while rho of tile k is held in registers
          for (int c0 = cbeg; c0 < cend; c0 += 16) {
            uint32_t mys = 0;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t s1[8], s2[8];
              tmem_ld8(dT1 + c0 + 8 * hh, s1);
              tmem_ld8(dT2 + c0 + 8 * hh, s2);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float sv = fmaf(__uint_as_float(s2[j]), kSplitScaleInv, __uint_as_float(s1[j]));
                const uint32_t w = __ballot_sync(0xffffffffu, active && sv >= 0.0f);
                if (lane == 8 * hh + j) mys = w;
              }
            }
            if (q < G && lane < 16) signs_stage[(c0 + lane) * G + q] = mys;
          }
          tc_fence_before();
        }
        if (has_tile) {
          // the rho buffer is free (the T rho products of tile k-1 are complete): store rho of tile k
          if (NV == 64) {
            if (i < KP) {
#pragma unroll
              for (int bt = 0; bt < (NV == 64 ? 2 : 1); ++bt) {
                const int c0 = cbeg + 16 * bt;
                const uint32_t o0 = sw128_offset(i, 2 * c0, 128), o1 = sw128_offset(i, 2 * c0 + 16, 128);
                *(uint4*)(rho_hi + o0) = make_uint4(rhw[bt][0], rhw[bt][1], rhw[bt][2], rhw[bt][3]);
                *(uint4*)(rho_hi + o1) = make_uint4(rhw[bt][4], rhw[bt][5], rhw[bt][6], rhw[bt][7]);
                *(uint4*)(rho_lo + o0) = make_uint4(rlw[bt][0], rlw[bt][1], rlw[bt][2], rlw[bt][3]);
                *(uint4*)(rho_lo + o1) = make_uint4(rlw[bt][4], rlw[bt][5], rlw[bt][6], rlw[bt][7]);
              }
            }
          } else if (i < KP) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint32_t off = sw128_offset(cbeg + j, 2 * i, NV);
              *(__half*)(rho_hi + off) = rhs[j];
              *(__half*)(rho_lo + off) = rls[j];
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[RHO_FULL]);
        }
      }
      if (!epi_sync()) break;
      if (has_tile) {
        uint32_t* dst = p.codes + v0 * wrec;
        const int nw = rows * wrec;
        for (int w = te; w < nw; w += 256) dst[w] = codes_stage[w];
        if (ALG2 && te < rows) {
          float g2 = 0.0f;
          for (int qq = 0; qq < G; ++qq) g2 += gpart[qq * NV + te];
          p.gammas[v0 + te] = __half_as_ushort(__float2half_rn(sqrtf(g2)));
        }
      }
      if (ALG2 && k >= 1) {
        uint32_t* dst = p.signs + v0p * G;
        const int nw = rowsp * G;
        for (int w = te; w < nw; w += 256) dst[w] = signs_stage[w];
      }
      if (!ALG2) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[ACC_EMPTY + a]);
          mbar_arrive(&bar[INFO_EMPTY + a]);
        }
      }
      v0p = v0;
      rowsp = rows;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, NCOLS);
  }
}

template <int XT, bool ALG2, int NV, int BITS>
tq_status launch_encode(EncodeParams& p, const void* x, cudaStream_t st) {
  constexpr int ES = XT == TQ_BF16 ? 2 : 4;
  const EncLayout Lo = enc_layout<XT, ALG2, NV, BITS == 0 ? 4 : BITS>(p.d, p.KP, p.G);
  alignas(64) CUtensorMap tmap;
  if (!make_tmap_2d_sw128(&tmap, x, ES, (uint64_t)p.d, (uint64_t)p.n, 128 / ES, NV))
    return fail(TQ_ERR_CUDA, "encode: could not create the TMA tensor map of x");
  auto kern = encode_kernel<XT, ALG2, NV, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "encode: shared memory attribute");
  p.ntiles = (int)((p.n + NV - 1) / NV);
  const int grid = std::min(p.ntiles, sm_count());
  kern<<<grid, enc_threads(ALG2, NV), Lo.total, st>>>(p, tmap);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "encode: launch");
  return TQ_OK;
}

template <int XT, bool ALG2, int NV>
tq_status launch_bits(EncodeParams& p, int bits, const void* x, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_encode<XT, ALG2, NV, 1>(p, x, st);
    case 2: return launch_encode<XT, ALG2, NV, 2>(p, x, st);
    case 3: return launch_encode<XT, ALG2, NV, 3>(p, x, st);
    default: return launch_encode<XT, ALG2, NV, 4>(p, x, st);
  }
}

tq_status encode_common(const char* fn, const tq_codebook* cb, int64_t n, int32_t d, const void* x, int32_t xt,
                        const void* rot, uint32_t* codes, uint32_t* signs, uint16_t* norms, uint16_t* gammas,
                        bool alg2, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  std::string f(fn);
  if (!cb || !rot || !codes || !norms || (n > 0 && !x)) return fail(TQ_ERR_INVALID_ARG, f + ": NULL pointer");
  if (alg2 && (!signs || !gammas)) return fail(TQ_ERR_INVALID_ARG, f + ": NULL signs / gammas");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, f + ": n < 0");
  if (!valid_dim(d)) return fail(TQ_ERR_UNSUPPORTED, f + ": d must be a multiple of 32 in [32, 4096]");
  if (cb->d != d || cb->bits < 1 || cb->bits > 4 || cb->levels != (1 << cb->bits))
    return fail(TQ_ERR_INVALID_ARG, f + ": codebook does not match d / has bad bits");
  const int L = cb->levels, H = L / 2;
  for (int k = 0; k < L; ++k)
    if (cb->c[L - 1 - k] != -cb->c[k]) return fail(TQ_ERR_INVALID_ARG, f + ": codebook is not symmetric");
  for (int k = 0; k + 1 < L; ++k)
    if (cb->t[L - 2 - k] != -cb->t[k]) return fail(TQ_ERR_INVALID_ARG, f + ": codebook is not symmetric");
  if (xt != TQ_F32 && xt != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, f + ": x_dtype must be TQ_F32 or TQ_BF16");
  if (!aligned16(x) || !aligned16(rot) || !aligned16(codes) || !aligned16(norms) ||
      (alg2 && (!aligned16(signs) || !aligned16(gammas))))
    return fail(TQ_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  if (n == 0) return TQ_OK;
  if (n > ((int64_t)1 << 31) - 256) return fail(TQ_ERR_UNSUPPORTED, f + ": n >= 2^31");
  if (d > 128) return encode_tiled(cb, n, d, x, xt, rot, codes, signs, norms, gammas, alg2, ws, ws_bytes, stream);
  RotLayout RL = rot_layout(d);
  const uint8_t* base = (const uint8_t*)rot;
  EncodeParams p{};
  p.n = n;
  p.d = d;
  p.G = d / 32;
  p.KP = d <= 64 ? 64 : 128;
  p.img[0] = base + RL.pi_hi;
  p.img[1] = base + RL.pi_lo;
  p.img[2] = base + RL.t_hi;
  p.img[3] = base + RL.t_lo;
  p.img_bytes = 128u * p.KP * 2;
  p.codes = codes;
  p.signs = signs;
  p.norms = norms;
  p.gammas = gammas;
  for (int k = 0; k < 8; ++k) {
    p.P[k] = k < H - 1 ? cb->t[H + k] : 0.0f;
    p.C[k] = k < H ? cb->c[H + k] : 0.0f;
  }
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, f + ": no device error word (is a CUDA device present?)");
  cudaStream_t st = (cudaStream_t)stream;
  if (!alg2)
    return xt == TQ_BF16 ? launch_bits<TQ_BF16, false, 128>(p, cb->bits, x, st)
                         : launch_bits<TQ_F32, false, 64>(p, cb->bits, x, st);
  return xt == TQ_BF16 ? launch_bits<TQ_BF16, true, 64>(p, cb->bits, x, st)
                       : launch_bits<TQ_F32, true, 32>(p, cb->bits, x, st);
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" TQ_API size_t tq_encode_workspace_bytes(int64_t n, int32_t d, int32_t alg) {
  if (n < 0 || (alg != 1 && alg != 2) || !valid_dim(d)) return 0;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      nsm <= 0) {
    cudaGetLastError();
    nsm = 148;
  }
  return encode_tiled_ws_bytes(n, d, alg == 2, nsm);
}

extern "C" TQ_API tq_status tq_encode_mse(const tq_codebook* cb, int64_t n, int32_t d, const void* x, int32_t x_dtype,
                                   const void* rot, uint32_t* codes, uint16_t* norms, void* stream) {
  return encode_common("tq_encode_mse", cb, n, d, x, x_dtype, rot, codes, nullptr, norms, nullptr, false, nullptr, 0,
                       stream);
}

extern "C" TQ_API tq_status tq_encode_prod(const tq_codebook* cb_bm1, int64_t n, int32_t d, const void* x, int32_t x_dtype,
                                    const void* rot, uint32_t* codes, uint32_t* signs, uint16_t* norms,
                                    uint16_t* gammas, void* ws, size_t ws_bytes, void* stream) {
  return encode_common("tq_encode_prod", cb_bm1, n, d, x, x_dtype, rot, codes, signs, norms, gammas, true, ws, ws_bytes,
                       stream);
}

// Algorithm 1 with a bit width per group of 32 rotated coordinates (d <= 128): each epilogue warp
// quantises one group with that group's codebook and writes its planes at the group's offset in the
// record.
extern "C" TQ_API tq_status tq_encode_mse_mixed(const tq_codebook* cbs, const int32_t* group_bits, int64_t n,
                                                int32_t d, const void* x, int32_t x_dtype, const void* rot,
                                                uint32_t* codes, uint16_t* norms, void* stream) {
  clear_error();
  const std::string f = "tq_encode_mse_mixed";
  if (!cbs || !group_bits || !rot || !codes || !norms || (n > 0 && !x)) return fail(TQ_ERR_INVALID_ARG, f + ": NULL pointer");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, f + ": n < 0");
  if (!valid_dim(d) || d > 128) return fail(TQ_ERR_UNSUPPORTED, f + ": d must be 32, 64, 96 or 128");
  const int G = d / 32;
  EncodeParams p{};
  int wv = 0;
  for (int g = 0; g < G; ++g) {
    const int b = group_bits[g];
    if (b < 1 || b > 4) return fail(TQ_ERR_UNSUPPORTED, f + ": group widths must be 1..4 bits");
    const tq_codebook* cb = &cbs[b - 1];
    if (cb->d != d || cb->bits != b || cb->levels != (1 << b))
      return fail(TQ_ERR_INVALID_ARG, f + ": cbs[b - 1] must be the b-bit codebook for this d");
    const int L = cb->levels, H = L / 2;
    for (int k = 0; k < L; ++k)
      if (cb->c[L - 1 - k] != -cb->c[k]) return fail(TQ_ERR_INVALID_ARG, f + ": codebook is not symmetric");
    p.gbits[g] = b;
    p.goff[g] = wv;
    wv += b;
    for (int k = 0; k < 8; ++k) p.Pm[g][k] = k < H - 1 ? cb->t[H + k] : 0.0f;
  }
  p.wv = wv;
  if (x_dtype != TQ_F32 && x_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, f + ": x_dtype must be TQ_F32 or TQ_BF16");
  if (!aligned16(x) || !aligned16(rot) || !aligned16(codes) || !aligned16(norms))
    return fail(TQ_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  if (n == 0) return TQ_OK;
  if (n > ((int64_t)1 << 31) - 256) return fail(TQ_ERR_UNSUPPORTED, f + ": n >= 2^31");
  RotLayout RL = rot_layout(d);
  const uint8_t* base = (const uint8_t*)rot;
  p.n = n;
  p.d = d;
  p.G = G;
  p.KP = d <= 64 ? 64 : 128;
  p.img[0] = base + RL.pi_hi;
  p.img[1] = base + RL.pi_lo;
  p.img[2] = base + RL.t_hi;
  p.img[3] = base + RL.t_lo;
  p.img_bytes = 128u * p.KP * 2;
  p.codes = codes;
  p.norms = norms;
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, f + ": no device error word (is a CUDA device present?)");
  cudaStream_t st = (cudaStream_t)stream;
  return x_dtype == TQ_BF16 ? launch_encode<TQ_BF16, false, 128, 0>(p, x, st) : launch_encode<TQ_F32, false, 64, 0>(p, x, st);
}
