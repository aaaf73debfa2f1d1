// Tiled TurboQuant encode for d > 128 (multiples of 128 up to 4096): Algorithm 1 and 2.
//
// Method as in the fused kernel (ai-navigate-news page, "how it works (technical)"; aiboss88
// page, "technical principles"): y = Pi x / |x|, idx_j = #{k : t_k < y_j}, bit planes of idx,
// fp16 |x|; Algorithm 2 adds rho = y - c[idx], gamma = |rho| and the signs of S r = T rho.
//
// Orientation: M = 128 vectors per tile (TMEM lane = vector), N = one 128-row band of output
// coordinates, K = 64-coordinate blocks. A tile is processed in sweeps over its K blocks:
//   sweep 0          the converter warps read x once and form |x| in fp64 (the power-of-two
//                    scale of the fp16 operands must be known before any conversion);
//   sweeps 1..NB     y for band nb: D_hi = x_hi Pi_hi^T, D_lo = x_hi Pi_lo^T (+ x_lo Pi_hi^T for
//                    fp32 input); the epilogue (thread = vector) quantises, packs its own bit-plane
//                    words (no ballots: a thread holds 32 consecutive coordinates), and for
//                    Algorithm 2 writes rho (scaled by 2^14, split hi + 2^-12 lo) into this CTA's
//                    workspace slot as tensor-core operand images and accumulates |rho|^2;
//   sweeps NB+1..2NB (Algorithm 2) s = T rho for band nb from the rho images (3 split
//                    products); the epilogue packs the sign words.
// The x tile is re-read from L2 in every sweep of the tile (it was read from HBM once).
// Precision: products exact in the tensor core, fp32 accumulation over K = d. For large d the
// accumulated rounding approaches the parity band, so a decision whose value lies within 20x the
// band of a boundary (a quantiser boundary, or zero for a sign) is recomputed exactly in fp64 from
// the fp32 matrices -- rare (below 1e-3 of the decisions at d = 1536) and off the fast path. The
// same holds for the fp16 rounding of gamma = |r|: a gamma within 2^-15 (relative) of an fp16
// rounding midpoint, far wider than the fp32 accumulation error, is flagged, and a fix-up kernel
// recomputes r = x / |x| - Pi^T c[idx] for that vector in fp64 from x, the fp32 Pi and the vector's
// own codes, and rewrites gamma (about 9 % of the vectors; d^2 fp64 operations each, one pass over
// Pi serving a batch of eight).
//
// Roles (10 warps): 0 TMA / bulk copies; 1 TMEM owner and MMA issuer; 2-5 converters (thread =
// vector: fp64 norm, fp16 split of x, copies of the rho images); 6-9 epilogue (thread = vector).
// All waits are bounded (sm100.cuh).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <string>

#include "quant_device.cuh"
#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kTThreads = 320;
constexpr float kRhoScaleT = 16384.0f;   // 2^14: |rho| < 2 keeps rho * 2^14 below the fp16 maximum
constexpr uint32_t kBlk = 16384;         // one operand block: 128 rows x 64 fp16 (128-byte swizzle)

struct TEParams {
  int64_t n;
  int d, G, KB, NB, ntiles;
  const uint8_t* pi_hi;
  const uint8_t* pi_lo;
  const uint8_t* t_hi;
  const uint8_t* t_lo;
  uint32_t band_bytes;       // bytes of one 128-row band of a rotation image
  uint32_t* codes;
  uint32_t* signs;
  uint16_t* norms;
  uint16_t* gammas;
  uint8_t* rho;              // per-CTA slots of slot_bytes: [KB][hi, lo][kBlk]
  size_t slot_bytes;
  uint32_t* gflag;           // one bit per vector: gamma next to an fp16 rounding midpoint (Algorithm 2)
  const void* x;             // the input (exact recomputation of decisions next to a boundary)
  const float* pi32;         // fp32 Pi, row-major
  const float* t32;          // fp32 T = S Pi^T, row-major
  const float* s32;          // fp32 S, row-major
  float P[8], C[8];
  uint32_t* err;
};

struct TLayout {
  uint32_t raw, a, b, info, bar, total;
};
__host__ __device__ inline TLayout t_layout() {
  TLayout L{};
  L.raw = 0;                       // [2][2 x kBlk]  raw x blocks (fp32: two 32-column boxes)
  L.a = L.raw + 4 * kBlk;          // [2][hi, lo]    fp16 A operand blocks
  L.b = L.a + 4 * kBlk;            // [2][hi, lo]    fp16 B operand blocks (Pi or T band blocks)
  L.info = L.b + 4 * kBlk;         // [2][128] float 1 / (|x| 2^e), then [2][128] double |x|, tile parity
  L.bar = L.info + 2 * 128 * 4 + 2 * 128 * 8;
  L.total = L.bar + 32 * 8 + 1024;
  return L;
}

enum TBars {
  RAW_FULL = 0, RAW_EMPTY = 2, B_FULL = 4, B_EMPTY = 6, A_FULL = 8, A_EMPTY = 10, ACC_FULL = 12, ACC_EMPTY = 14,
  NORM_READY = 16, INFO_EMPTY = 18, RHO_READY = 20, TNBARS = 21
};

// P[k] for 0 <= k < H - 1, as a tree of selects on the bits of k: with no indexed access to P the
// compiler keeps the boundaries in registers (an indexed form placed them in local memory).
template <int BITS>
__device__ __forceinline__ float sym_p(int k, const float (&P)[8]) {
  if (BITS <= 2) return P[0];
  if (BITS == 3) return (k & 2) ? P[2] : ((k & 1) ? P[1] : P[0]);
  const float lo = (k & 2) ? ((k & 1) ? P[3] : P[2]) : ((k & 1) ? P[1] : P[0]);
  const float hi = (k & 2) ? P[6] : ((k & 1) ? P[5] : P[4]);
  return (k & 4) ? hi : lo;
}

// Cell of |y| the symmetric quantiser chose: (lo, hi] with lo = P[m-1] (0 for m = 0), hi = P[m]
// (infinity for the top cell).
template <int BITS>
__device__ __forceinline__ void sym_bounds(int m, const float (&P)[8], float& lo, float& hi) {
  constexpr int H = 1 << (BITS - 1);
  lo = m == 0 ? 0.0f : sym_p<BITS>(m - 1, P);
  hi = m == H - 1 ? INFINITY : sym_p<BITS>(m, P);
}

// Exact (fp64) recomputation of a decision whose fp32 tensor-core value lies next to a boundary:
// y_i = (Pi x)_i / |x| for a code, and for a sign (S r)_j for r = x / |x| - Pi^T c[idx], evaluated
// as (S x)_j / |x| - (T c[idx])_j from the fp32 S and T and the vector's own codes (already
// written). Rare: only values within 20x the parity band of a boundary take this path.
// Both are computed by a whole warp for one lane's vector: each lane sums a strided slice of the d
// terms in fp64, then a butterfly sum leaves the same total in every lane, so a decision next to a
// boundary costs the warp d / 32 terms per lane instead of d serial terms.
template <bool F32>
__device__ __noinline__ double warp_row_dot_x(const float* prow, const void* x, int64_t v, int d, int lane) {
  double a0 = 0.0, a1 = 0.0;
  for (int k = lane; k < d; k += 64) {
    const int k1 = k + 32;
    if (F32) {
      const float* xr = (const float*)x + v * d;
      a0 = fma((double)__ldg(prow + k), (double)__ldg(xr + k), a0);
      if (k1 < d) a1 = fma((double)__ldg(prow + k1), (double)__ldg(xr + k1), a1);
    } else {
      const unsigned short* xr = (const unsigned short*)x + v * d;
      a0 = fma((double)__ldg(prow + k), (double)__uint_as_float((uint32_t)__ldg(xr + k) << 16), a0);
      if (k1 < d) a1 = fma((double)__ldg(prow + k1), (double)__uint_as_float((uint32_t)__ldg(xr + k1) << 16), a1);
    }
  }
  double s = a0 + a1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

template <bool F32, int BITS>
__device__ __noinline__ double warp_sign_value(const float* srow, const float* trow, const void* x, int64_t v, int d,
                                               double nrm, const uint32_t* vcodes, const float* C, int lane) {
  const double sx = warp_row_dot_x<F32>(srow, x, v, d, lane) / nrm;
  constexpr int H = 1 << (BITS - 1);
  double tc = 0.0;
  for (int k = lane; k < d; k += 32) {              // coordinate k = 32 (k >> 5) + lane of the code words
    const uint32_t* wk = vcodes + (k >> 5) * BITS;
    const bool neg = ((wk[BITS - 1] >> lane) & 1u) == 0u;
    int m = 0;
    for (int pl = 0; pl < BITS - 1; ++pl) m |= (int)((wk[pl] >> lane) & 1u) << pl;
    if (neg) m ^= H - 1;
    const float cm = C[m];
    tc = fma((double)__ldg(trow + k), neg ? -(double)cm : (double)cm, tc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tc += __shfl_xor_sync(0xffffffffu, tc, o);
  return sx - tc;
}

constexpr double kGammaFixTol = 1.0 / 32768.0;   // 2^-15: flag gamma this close to an fp16 midpoint

// True when x > 0 lies within tol (relative) of the midpoint between its fp16 rounding and the
// neighbouring fp16 value on x's side, i.e. where a small error in x could flip the rounding.
__device__ __forceinline__ bool near_f16_midpoint(double x, double tol) {
  const __half h = __double2half(x);
  const double hd = (double)__half2float(h);
  const unsigned short hb = __half_as_ushort(h);
  if (hb >= 0x7BFFu) return false;                       // at or past the largest finite value
  const unsigned short nb = (x >= hd) ? (unsigned short)(hb + 1u) : (hb == 0u ? hb : (unsigned short)(hb - 1u));
  const double mid = 0.5 * (hd + (double)__half2float(__ushort_as_half(nb)));
  return fabs(x - mid) <= tol * x;
}

constexpr int kFixThreads = 256;
constexpr size_t kFixCounterBytes = 16;          // the fix-up's claim counter, after the flag words
constexpr int kFixChunkWords = 4;                // flag words (128 vectors) a block claims at a time

// Exact gamma for the flagged vectors: r = x / |x| - Pi^T c[idx] in fp64 (original domain, the
// vector's own codes), gamma = |r| rounded to fp16. Blocks claim chunks of flag words from a
// counter that follows the flag words, and take the flagged vectors VB at a time: one pass over the
// fp32 Pi serves the whole batch (Pi is read once per VB vectors) and every thread keeps 2 x VB
// independent fp64 sums in flight. For each vector the sums are formed in the order of a plain
// one-vector loop: (Pi^T c)_j = sum over i ascending, |x|^2 and |r|^2 over this thread's columns
// j = tid + 256 t ascending, then a warp butterfly and the warps' totals in warp order.
template <bool F32, int BITS, int VB>
__global__ void __launch_bounds__(kFixThreads) gamma_fixup_kernel(const __grid_constant__ TEParams p, int nwords) {
  extern __shared__ __align__(16) double cs[];        // [d][VB]: c_i of the batch's vectors (fp64)
  __shared__ double red[kFixThreads / 32][VB];
  __shared__ double nrm_s[VB];
  __shared__ int64_t vsel[VB];
  __shared__ int nsel;
  constexpr int NW = kFixThreads / 32, H = 1 << (BITS - 1);
  const int d = p.d, G = p.G, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned int* counter = (unsigned int*)(p.gflag + nwords);
  auto xval = [&](int64_t v, int j) -> double {
    return F32 ? (double)((const float*)p.x)[v * d + j]
               : (double)__uint_as_float((uint32_t)((const uint16_t*)p.x)[v * d + j] << 16);
  };
  // totals of VB per-thread values over the block (every thread gets them; red is free afterwards)
  auto block_sums = [&](double (&v)[VB], double (&out)[VB]) {
#pragma unroll
    for (int k = 0; k < VB; ++k) {
      double t = v[k];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      if (lane == 0) red[warp][k] = t;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < VB; ++k) {
      double t = 0.0;
#pragma unroll
      for (int w = 0; w < NW; ++w) t += red[w][k];
      out[k] = t;
    }
    __syncthreads();
  };
  // thread 0's cursor over the claimed flag words
  int cur = 0, cend = 0, wbase = 0;
  uint32_t bits = 0u;
  bool drained = false;
  for (;;) {
    __syncthreads();                                  // the previous batch's vsel / nsel are read
    if (tid == 0) {
      int n = 0;
      while (n < VB && !drained) {
        if (bits) {
          vsel[n++] = (int64_t)wbase * 32 + (__ffs(bits) - 1);
          bits &= bits - 1u;
        } else if (cur < cend) {
          wbase = cur;
          bits = p.gflag[cur++];
        } else {
          const int c = (int)atomicAdd(counter, 1u) * kFixChunkWords;
          if (c >= nwords) {
            drained = true;
          } else {
            cur = c;
            cend = min(nwords, c + kFixChunkWords);
          }
        }
      }
      nsel = n;
    }
    __syncthreads();
    const int n = nsel;
    if (n == 0) break;
    // |x| of the batch
    double acc[VB], tot[VB];
#pragma unroll
    for (int k = 0; k < VB; ++k) acc[k] = 0.0;
    for (int j = tid; j < d; j += kFixThreads) {
#pragma unroll
      for (int k = 0; k < VB; ++k)
        if (k < n) {
          const double xj = xval(vsel[k], j);
          acc[k] = fma(xj, xj, acc[k]);
        }
    }
    block_sums(acc, tot);
#pragma unroll
    for (int k = 0; k < VB; ++k)
      if (tid == k) nrm_s[k] = sqrt(tot[k]);
    // c[idx] of the batch from its code words
    for (int i = tid; i < d; i += kFixThreads) {
      const int l = i & 31;
#pragma unroll
      for (int k = 0; k < VB; ++k) {
        double c = 0.0;
        if (k < n) {
          const uint32_t* wk = p.codes + (size_t)vsel[k] * G * BITS + (i >> 5) * BITS;
          const bool neg = ((wk[BITS - 1] >> l) & 1u) == 0u;
          int m = 0;
          for (int pl = 0; pl < BITS - 1; ++pl) m |= (int)((wk[pl] >> l) & 1u) << pl;
          if (neg) m ^= H - 1;
          float cm = p.C[0];
#pragma unroll
          for (int q = 1; q < H; ++q)
            if (q == m) cm = p.C[q];
          c = neg ? -(double)cm : (double)cm;
        }
        cs[(size_t)i * VB + k] = c;
      }
    }
    __syncthreads();
    // r_j = x_j / |x| - (Pi^T c)_j for this thread's columns, two at a time
#pragma unroll
    for (int k = 0; k < VB; ++k) acc[k] = 0.0;         // |r|^2
    for (int j0 = tid; j0 < d; j0 += 2 * kFixThreads) {
      const int j1 = j0 + kFixThreads;
      const bool h1 = j1 < d;
      double a0[VB], a1[VB];
#pragma unroll
      for (int k = 0; k < VB; ++k) a0[k] = a1[k] = 0.0;
      const float* p0 = p.pi32 + j0;
      const float* p1 = p.pi32 + (h1 ? j1 : j0);
#pragma unroll 4
      for (int i = 0; i < d; ++i) {
        const double pi0 = (double)__ldg(p0 + (size_t)i * d);
        const double pi1 = (double)__ldg(p1 + (size_t)i * d);
        const double2* cv = (const double2*)(cs + (size_t)i * VB);
#pragma unroll
        for (int kk = 0; kk < VB / 2; ++kk) {
          const double2 c2 = cv[kk];
          a0[2 * kk] = fma(pi0, c2.x, a0[2 * kk]);
          a0[2 * kk + 1] = fma(pi0, c2.y, a0[2 * kk + 1]);
          a1[2 * kk] = fma(pi1, c2.x, a1[2 * kk]);
          a1[2 * kk + 1] = fma(pi1, c2.y, a1[2 * kk + 1]);
        }
      }
#pragma unroll
      for (int k = 0; k < VB; ++k)
        if (k < n) {
          const double nk = nrm_s[k];
          const double r0 = xval(vsel[k], j0) / nk - a0[k];
          acc[k] = fma(r0, r0, acc[k]);
          if (h1) {
            const double r1 = xval(vsel[k], j1) / nk - a1[k];
            acc[k] = fma(r1, r1, acc[k]);
          }
        }
    }
    block_sums(acc, tot);
#pragma unroll
    for (int k = 0; k < VB; ++k)
      if (tid == k && k < n) p.gammas[vsel[k]] = __half_as_ushort(__double2half(sqrt(tot[k])));
  }
}

// Fix-up batch size: the batch's fp64 codebook values (d x VB) must fit in shared memory.
inline int fixup_batch(int d) { return d <= 3072 ? 8 : 4; }

template <bool F32, bool ALG2, int BITS>
__global__ void __launch_bounds__(kTThreads, 1)
    encode_tiled_kernel(const __grid_constant__ TEParams p, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const TLayout Lo = t_layout();
  uint64_t* bar = (uint64_t*)(smem + Lo.bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + TNBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + TNBARS) + 1;
  float* info = (float*)(smem + Lo.info);
  double* nrmd = (double*)(smem + Lo.info + 2 * 128 * 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = p.KB, NB = p.NB, G = p.G;
  const int nsweeps = 1 + NB + (ALG2 ? NB : 0);
  __shared__ float c_tab[8];                 // the positive centroids, for the exact sign fallback
  if (tid < 8) c_tab[tid] = p.C[tid];

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[RAW_FULL + s], 1);
      mbar_init(&bar[RAW_EMPTY + s], 4);
      mbar_init(&bar[B_FULL + s], 1);
      mbar_init(&bar[B_EMPTY + s], 1);
      mbar_init(&bar[A_FULL + s], 4);
      mbar_init(&bar[A_EMPTY + s], 1);
      mbar_init(&bar[ACC_FULL + s], 1);
      mbar_init(&bar[ACC_EMPTY + s], 4);
      mbar_init(&bar[NORM_READY + s], 4);
      mbar_init(&bar[INFO_EMPTY + s], 4);
    }
    mbar_init(&bar[RHO_READY], 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  uint8_t* slot = p.rho ? p.rho + (size_t)blockIdx.x * p.slot_bytes : nullptr;

  if (warp == 0) {
    // ------------------------------------ producer -------------------------------------------------
    // warp-uniform schedule; one elected lane issues the copies
    uint32_t jr = 0, jb = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x) {
      for (int s = 0; s < nsweeps && ok; ++s) {
        const bool phase2 = s > NB;
        const int nb = phase2 ? s - 1 - NB : s - 1;
        for (int kb = 0; kb < KB; ++kb) {
          if (s <= NB) {
            const int rs = jr & 1;
            if (!mbar_wait_warp(&bar[RAW_EMPTY + rs], ((jr >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* dst = smem + Lo.raw + rs * 2 * kBlk;
            if (elect_one_sync()) {
              mbar_arrive_expect_tx(&bar[RAW_FULL + rs], F32 ? 2 * kBlk : kBlk);
              tma_load_2d(dst, &tmap, kb * 64, tile * 128, &bar[RAW_FULL + rs]);
              if (F32) tma_load_2d(dst + kBlk, &tmap, kb * 64 + 32, tile * 128, &bar[RAW_FULL + rs]);
            }
            __syncwarp();
            ++jr;
          }
          if (s >= 1) {
            const int bs = jb & 1;
            if (!mbar_wait_warp(&bar[B_EMPTY + bs], ((jb >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) {
              ok = false;
              break;
            }
            const size_t off = (size_t)nb * p.band_bytes + (size_t)kb * kBlk;
            uint8_t* dst = smem + Lo.b + bs * 2 * kBlk;
            if (elect_one_sync()) {
              mbar_arrive_expect_tx(&bar[B_FULL + bs], 2 * kBlk);
              bulk_g2s(dst, (phase2 ? p.t_hi : p.pi_hi) + off, kBlk, &bar[B_FULL + bs]);
              bulk_g2s(dst + kBlk, (phase2 ? p.t_lo : p.pi_lo) + off, kBlk, &bar[B_FULL + bs]);
            }
            __syncwarp();
            ++jb;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------ MMA issuer -----------------------------------------------
    // warp-uniform schedule (descriptors stay in uniform registers); one elected lane issues
    const uint32_t idesc = idesc_f16_f32(128, 128);
    const uint64_t da0 = desc_kmajor_sw128(smem_u32(smem + Lo.a));
    const uint64_t db0 = desc_kmajor_sw128(smem_u32(smem + Lo.b));
    uint32_t ja = 0, jb = 0, jacc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x) {
      for (int s = 1; s < nsweeps && ok; ++s) {
        const bool has_lo = F32 || s > NB;        // fp32 x or the rho operand carry a low part
        const int acc = jacc & 1;
        if (jacc >= 2 &&
            !mbar_wait_warp(&bar[ACC_EMPTY + acc], ((jacc >> 1) - 1) & 1, p.err, kDevTimeoutSync, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dhi = tbase + acc * 256, dlo = dhi + 128;
        for (int kb = 0; kb < KB; ++kb) {
          const int as = ja & 1, bs = jb & 1;
          if (!mbar_wait_warp(&bar[A_FULL + as], (ja >> 1) & 1, p.err, kDevTimeoutSync, abort_flag) ||
              !mbar_wait_warp(&bar[B_FULL + bs], (jb >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ah = da0 + ((as * 2 * kBlk) >> 4), al = ah + (kBlk >> 4);
          const uint64_t bh = db0 + ((bs * 2 * kBlk) >> 4), bl = bh + (kBlk >> 4);
          if (elect_one_sync()) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint32_t accum = (kb > 0 || ks > 0) ? 1u : 0u;
              mma_f16_ss(dhi, ah + 2 * ks, bh + 2 * ks, idesc, accum);
              mma_f16_ss(dlo, ah + 2 * ks, bl + 2 * ks, idesc, accum);
              if (has_lo) mma_f16_ss(dlo, al + 2 * ks, bh + 2 * ks, idesc, 1u);
            }
            mma_commit(&bar[A_EMPTY + as]);
            mma_commit(&bar[B_EMPTY + bs]);
          }
          __syncwarp();
          ++ja;
          ++jb;
        }
        if (ok && elect_one_sync()) mma_commit(&bar[ACC_FULL + acc]);
        __syncwarp();
        ++jacc;
      }
    }
  } else if (warp < 6) {
    // ------------------------------------ converters (thread = vector) -----------------------------
    const int r = (warp - 2) * 32 + lane;
    uint32_t jr = 0, ja = 0;
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x, ++tl) {
      const int64_t v = (int64_t)tile * 128 + r;
      const bool live = v < p.n;
      // sweep 0: |x| in fp64
      double ss = 0.0;
      for (int kb = 0; kb < KB; ++kb) {
        const int rs = jr & 1;
        if (!mbar_wait_warp(&bar[RAW_FULL + rs], (jr >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* raw = smem + Lo.raw + rs * 2 * kBlk;
        if (F32) {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float4 f = *(const float4*)(raw + (c >> 3) * kBlk + sw128_offset(r, (c & 7) * 16, 128));
            ss = fma((double)f.x, (double)f.x, ss);
            ss = fma((double)f.y, (double)f.y, ss);
            ss = fma((double)f.z, (double)f.z, ss);
            ss = fma((double)f.w, (double)f.w, ss);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 w = *(const uint4*)(raw + sw128_offset(r, c * 16, 128));
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const double a = (double)__uint_as_float(u[k] << 16), b = (double)__uint_as_float(u[k] & 0xFFFF0000u);
              ss = fma(a, a, ss);
              ss = fma(b, b, ss);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[RAW_EMPTY + rs]);
        ++jr;
      }
      if (!ok) break;
      const double nrm = sqrt(ss);
      float f1 = 1.0f, f2 = 1.0f, inv = 0.0f;
      if (nrm > 0.0) {
        int E;
        frexp(nrm, &E);
        pow2_pair(15 - E, f1, f2);                   // |x| f1 f2 in [2^14, 2^15)
        inv = (float)(1.0 / ldexp(nrm, 15 - E));
      }
      const int it = tl & 1;
      if (tl >= 2 && !mbar_wait_warp(&bar[INFO_EMPTY + it], ((tl >> 1) - 1) & 1, p.err, kDevTimeoutSync, abort_flag))
        break;
      info[it * 128 + r] = inv;
      nrmd[it * 128 + r] = nrm;
      if (live) p.norms[v] = __half_as_ushort(__double2half(nrm));
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[NORM_READY + it]);
      // sweeps 1..NB: fp16 split of x f1 f2 into the A ring
      for (int nb = 0; nb < NB && ok; ++nb) {
        for (int kb = 0; kb < KB; ++kb) {
          const int rs = jr & 1, as = ja & 1;
          if (!mbar_wait_warp(&bar[RAW_FULL + rs], (jr >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag) ||
              (ja >= 2 && !mbar_wait_warp(&bar[A_EMPTY + as], ((ja >> 1) - 1) & 1, p.err, kDevTimeoutMma, abort_flag))) {
            ok = false;
            break;
          }
          const uint8_t* raw = smem + Lo.raw + rs * 2 * kBlk;
          uint8_t* ah = smem + Lo.a + as * 2 * kBlk;
#pragma unroll
          for (int c = 0; c < 8; ++c) {                // output chunk c: elements 8c .. 8c+7
            uint4 wh, wl = make_uint4(0, 0, 0, 0);
            if (F32) {
              const float4 fa = *(const float4*)(raw + (c >> 2) * kBlk + sw128_offset(r, ((2 * c) & 7) * 16, 128));
              const float4 fb = *(const float4*)(raw + (c >> 2) * kBlk + sw128_offset(r, ((2 * c + 1) & 7) * 16, 128));
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
            } else {
              const uint4 w = *(const uint4*)(raw + sw128_offset(r, c * 16, 128));
              auto cvt = [&](uint32_t u) -> uint32_t {
                return h2_bits(__floats2half2_rn(__uint_as_float(u << 16) * f1 * f2,
                                                 __uint_as_float(u & 0xFFFF0000u) * f1 * f2));
              };
              wh = make_uint4(cvt(w.x), cvt(w.y), cvt(w.z), cvt(w.w));
            }
            const uint32_t off = sw128_offset(r, c * 16, 128);
            *(uint4*)(ah + off) = wh;
            if (F32) *(uint4*)(ah + kBlk + off) = wl;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar[A_FULL + as]);
            mbar_arrive(&bar[RAW_EMPTY + rs]);
          }
          ++jr;
          ++ja;
        }
      }
      if (!ok) break;
      if (ALG2) {
        // sweeps NB+1..2NB: the A operand is the rho image the epilogue wrote for this tile
        if (!mbar_wait_warp(&bar[RHO_READY], tl & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        for (int nb = 0; nb < NB && ok; ++nb) {
          for (int kb = 0; kb < KB; ++kb) {
            const int as = ja & 1;
            // all sixteen loads of this thread's row go out before the stage wait and the stores
            // (interleaved, each store waited for its load: one L2 round trip per 32 bytes)
            const uint8_t* src = slot + (size_t)kb * 2 * kBlk;
            uint4 vh[8], vl[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t off = sw128_offset(r, c * 16, 128);
              vh[c] = __ldcg((const uint4*)(src + off));
              vl[c] = __ldcg((const uint4*)(src + kBlk + off));
            }
            if (ja >= 2 && !mbar_wait_warp(&bar[A_EMPTY + as], ((ja >> 1) - 1) & 1, p.err, kDevTimeoutMma, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t* ah = smem + Lo.a + as * 2 * kBlk;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t off = sw128_offset(r, c * 16, 128);
              *(uint4*)(ah + off) = vh[c];
              *(uint4*)(ah + kBlk + off) = vl[c];
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[A_FULL + as]);
            ++ja;
          }
        }
      }
    }
  } else {
    // ------------------------------------ epilogue (thread = vector) -------------------------------
    const int q = warp & 3;                       // TMEM lane quarter
    const int r = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    float P[8], C[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      P[k] = p.P[k];
      C[k] = p.C[k];
    }
    uint32_t jacc = 0;
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.ntiles && ok; tile += gridDim.x, ++tl) {
      const int64_t v = (int64_t)tile * 128 + r;
      const bool live = v < p.n;
      const int it = tl & 1;
      if (!mbar_wait_warp(&bar[NORM_READY + it], (tl >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
      const float inv = info[it * 128 + r];
      const double nrm = nrmd[it * 128 + r];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[INFO_EMPTY + it]);
      double g2 = 0.0;                              // |rho|^2 over d coordinates, fp64
      const float tau_y = 2e-4f * rsqrtf((float)p.d);   // 20x the band (1e-5 on sqrt(d) y)
      for (int nb = 0; nb < NB; ++nb) {
        const int acc = jacc & 1;
        if (!mbar_wait_warp(&bar[ACC_FULL + acc], (jacc >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the 4 x BITS words of this band are contiguous in the vector's record: group g's BITS
        // plane words at g BITS. The loops over groups and over 8-coordinate chunks stay rolled:
        // fully unrolled, the epilogue's code outgrew the instruction cache.
        uint32_t* dst = p.codes + (live ? ((size_t)v * G + 4 * nb) * BITS : 0);
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
          uint32_t words[BITS];
#pragma unroll
          for (int pl = 0; pl < BITS; ++pl) words[pl] = 0u;
          const int i0 = nb * 128 + g * 32;
#pragma unroll 1
          for (int kq = 0; kq < 4; ++kq) {              // coordinates i0 + 8 kq .. + 7
            uint32_t hi[8], lo[8];
            const uint32_t col = tbase + lane_base + acc * 256 + g * 32 + 8 * kq;
            tmem_ld8(col, hi);
            tmem_ld8(col + 128, lo);
            tmem_ld_wait();
            float rho[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int j = 8 * kq + jj;
              float y = fmaf(__uint_as_float(lo[jj]), kSplitScaleInv, __uint_as_float(hi[jj])) * inv;
              bool neg = !(y > 0.0f);
              int m = sym_m<BITS>(fabsf(y), P);
              {
                float blo, bhi;
                sym_bounds<BITS>(m, P, blo, bhi);
                const float a = fabsf(y);
                // next to a boundary: decide on the fp64 value, computed by the whole warp for each
                // lane that needs one (coordinate i is the same for every lane)
                uint32_t nm = __ballot_sync(0xffffffffu, live && inv != 0.0f && fminf(a - blo, bhi - a) < tau_y);
                if (nm) {
                  const int i = i0 + j;
                  const float* prow = p.pi32 + (size_t)i * p.d;
                  while (nm) {
                    const int L = __ffs(nm) - 1;
                    nm &= nm - 1;
                    const double dot = warp_row_dot_x<F32>(prow, p.x, __shfl_sync(0xffffffffu, v, L), p.d, lane);
                    if (lane == L) {
                      const double yd = dot / nrm;
                      neg = !(yd > 0.0);
                      const double ad = fabs(yd);
                      int mm = 0;
#pragma unroll
                      for (int k = 0; k < (1 << (BITS - 1)) - 1; ++k) mm += (double)P[k] < ad ? 1 : 0;
                      m = mm;
                      y = (float)yd;
                    }
                  }
                }
              }
#pragma unroll
              for (int pl = 0; pl < BITS; ++pl) {
                const bool bit = pl == BITS - 1 ? !neg : ((((m >> pl) & 1) != 0) != neg);
                words[pl] |= (bit ? 1u : 0u) << j;
              }
              if (ALG2) {
                const float cm = sym_c<BITS>(m, C);
                float rr = neg ? y + cm : y - cm;
                if (inv == 0.0f) rr = 0.0f;
                g2 = fma((double)rr, (double)rr, g2);
                rho[jj] = rr;
              }
            }
            if (ALG2) {
              // rho * 2^14 as hi + 2^-12 lo fp16 into the rho image (block i0 / 64, 16 bytes at
              // element (i0 mod 64) + 8 kq of this vector's row)
              uint8_t* blk = slot + (size_t)(i0 >> 6) * 2 * kBlk;
              uint32_t h[4], l[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float a = rho[2 * u] * kRhoScaleT, b = rho[2 * u + 1] * kRhoScaleT;
                const __half2 hh = __floats2half2_rn(a, b);
                const float2 back = __half22float2(hh);
                h[u] = h2_bits(hh);
                l[u] = h2_bits(__floats2half2_rn((a - back.x) * kSplitScale, (b - back.y) * kSplitScale));
              }
              const uint32_t off = sw128_offset(r, (((i0 & 63) >> 3) + kq) * 16, 128);
              *(uint4*)(blk + off) = make_uint4(h[0], h[1], h[2], h[3]);
              *(uint4*)(blk + kBlk + off) = make_uint4(l[0], l[1], l[2], l[3]);
            }
          }
          if (live) {
#pragma unroll
            for (int pl = 0; pl < BITS; ++pl) dst[g * BITS + pl] = words[pl];
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[ACC_EMPTY + acc]);
        ++jacc;
      }
      if (!ok) break;
      if (ALG2) {
        __threadfence_block();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[RHO_READY]);
        const float tau_s = 2e-4f * (float)sqrt(g2) * kRhoScaleT;   // 20x the band (1e-5 of |r|), in 2^14 s units
        for (int nb = 0; nb < NB; ++nb) {
          const int acc = jacc & 1;
          if (!mbar_wait_warp(&bar[ACC_FULL + acc], (jacc >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int g = 0; g < 4; ++g) {
            uint32_t w = 0;
#pragma unroll 1
            for (int kq = 0; kq < 4; ++kq) {            // coordinates g 32 + 8 kq .. + 7 of the band
              uint32_t hi[8], lo[8];
              const uint32_t col = tbase + lane_base + acc * 256 + g * 32 + 8 * kq;
              tmem_ld8(col, hi);
              tmem_ld8(col + 128, lo);
              tmem_ld_wait();
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) {
                const int j = 8 * kq + jj;
                const float sv = fmaf(__uint_as_float(lo[jj]), kSplitScaleInv, __uint_as_float(hi[jj]));
                bool bit = sv >= 0.0f;
                // next to zero: decide on the exact fp64 value (the residual's own rounding
                // included), computed by the whole warp for each lane that needs one
                uint32_t nm = __ballot_sync(0xffffffffu, live && fabsf(sv) < tau_s);
                if (nm) {
                  const int jg = nb * 128 + g * 32 + j;
                  while (nm) {
                    const int L = __ffs(nm) - 1;
                    nm &= nm - 1;
                    const int64_t vl = __shfl_sync(0xffffffffu, v, L);
                    const double val = warp_sign_value<F32, BITS>(
                        p.s32 + (size_t)jg * p.d, p.t32 + (size_t)jg * p.d, p.x, vl, p.d,
                        __shfl_sync(0xffffffffu, nrm, L), p.codes + (size_t)vl * G * BITS, c_tab, lane);
                    if (lane == L) bit = val >= 0.0;
                  }
                }
                w |= (bit ? 1u : 0u) << j;
              }
            }
            if (live) p.signs[(size_t)v * G + 4 * nb + g] = w;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[ACC_EMPTY + acc]);
          ++jacc;
        }
        if (!ok) break;
        if (live) {
          const double gam = sqrt(g2);
          p.gammas[v] = __half_as_ushort(__double2half(gam));
          if (gam > 0.0 && near_f16_midpoint(gam, kGammaFixTol)) atomicOr(p.gflag + (v >> 5), 1u << (v & 31));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

template <bool F32, bool ALG2, int BITS>
tq_status launch_tiled(TEParams& p, const void* x, int grid, cudaStream_t st) {
  constexpr int ES = F32 ? 4 : 2;
  alignas(64) CUtensorMap tmap;
  if (!make_tmap_2d_sw128(&tmap, x, ES, (uint64_t)p.d, (uint64_t)p.n, 128 / ES, 128))
    return fail(TQ_ERR_CUDA, "encode: could not create the TMA tensor map of x");
  auto kern = encode_tiled_kernel<F32, ALG2, BITS>;
  const TLayout Lo = t_layout();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "encode: shared memory attribute");
  const int nwords = (int)((p.n + 31) / 32);
  if (ALG2 && (e = cudaMemsetAsync(p.gflag, 0, (size_t)nwords * 4 + kFixCounterBytes, st)) != cudaSuccess)
    return cuda_fail(e, "encode: clear the gamma flags");
  kern<<<grid, kTThreads, Lo.total, st>>>(p, tmap);
  if (ALG2) {
    const int vb = fixup_batch(p.d);
    auto fix = vb == 8 ? gamma_fixup_kernel<F32, BITS, 8> : gamma_fixup_kernel<F32, BITS, 4>;
    const int fsm = p.d * vb * (int)sizeof(double);
    if (fsm > 48 * 1024 && (e = cudaFuncSetAttribute(fix, cudaFuncAttributeMaxDynamicSharedMemorySize, fsm)) != cudaSuccess)
      return cuda_fail(e, "encode: gamma fix-up shared memory attribute");
    const int nchunks = (nwords + kFixChunkWords - 1) / kFixChunkWords;
    fix<<<std::max(1, std::min(nchunks, 2 * sm_count())), kFixThreads, fsm, st>>>(p, nwords);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "encode: launch");
  return TQ_OK;
}

template <bool F32, bool ALG2>
tq_status launch_tiled_bits(TEParams& p, int bits, const void* x, int grid, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_tiled<F32, ALG2, 1>(p, x, grid, st);
    case 2: return launch_tiled<F32, ALG2, 2>(p, x, grid, st);
    case 3: return launch_tiled<F32, ALG2, 3>(p, x, grid, st);
    default: return launch_tiled<F32, ALG2, 4>(p, x, grid, st);
  }
}

}  // namespace

// Algorithm 2 workspace: the residual slots of the tiles in flight (one per CTA), then one flag bit
// per vector (gamma next to an fp16 rounding midpoint), then the fix-up's claim counter.
size_t tiled_rho_bytes(int64_t n, int d, int nsm) {
  const int64_t ntiles = (n + 127) / 128;
  const int64_t grid = std::min<int64_t>(ntiles, nsm);
  return (size_t)grid * (size_t)(d / 64) * 2 * kBlk;
}

size_t encode_tiled_ws_bytes(int64_t n, int d, bool alg2, int nsm) {
  if (!alg2 || d <= 128 || n <= 0) return 0;
  return tiled_rho_bytes(n, d, nsm) + (size_t)((n + 31) / 32) * 4 + kFixCounterBytes;
}

tq_status encode_tiled(const tq_codebook* cb, int64_t n, int d, const void* x, int xt, const void* rot,
                       uint32_t* codes, uint32_t* signs, uint16_t* norms, uint16_t* gammas, bool alg2, void* ws,
                       size_t ws_bytes, void* stream) {
  const char* f = alg2 ? "tq_encode_prod" : "tq_encode_mse";
  if (d % 128) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": d > 128 must be a multiple of 128");
  const int nsm = sm_count();
  const size_t need = encode_tiled_ws_bytes(n, d, alg2, nsm);
  if (need > 0 && (!ws || ws_bytes < need)) return fail(TQ_ERR_WORKSPACE, std::string(f) + ": workspace too small");
  if (need > 0 && !aligned16(ws)) return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": workspace must be 16-byte aligned");
  const RotLayout RL = rot_layout(d);
  const uint8_t* base = (const uint8_t*)rot;
  TEParams p{};
  p.n = n;
  p.d = d;
  p.G = d / 32;
  p.KB = d / 64;
  p.NB = d / 128;
  p.ntiles = (int)((n + 127) / 128);
  p.pi_hi = base + RL.pi_hi;
  p.pi_lo = base + RL.pi_lo;
  p.t_hi = base + RL.t_hi;
  p.t_lo = base + RL.t_lo;
  p.band_bytes = (uint32_t)(128u * RL.dp * 2u);
  p.codes = codes;
  p.signs = signs;
  p.norms = norms;
  p.gammas = gammas;
  p.rho = alg2 ? (uint8_t*)ws : nullptr;
  p.gflag = alg2 ? (uint32_t*)((uint8_t*)ws + tiled_rho_bytes(n, d, nsm)) : nullptr;
  p.x = x;
  p.pi32 = (const float*)(base + RL.pi32);
  p.t32 = (const float*)(base + RL.t32);
  p.s32 = (const float*)(base + RL.s32);
  p.slot_bytes = (size_t)p.KB * 2 * kBlk;
  const int L = cb->levels, H = L / 2;
  for (int k = 0; k < 8; ++k) {
    p.P[k] = k < H - 1 ? cb->t[H + k] : 0.0f;
    p.C[k] = k < H ? cb->c[H + k] : 0.0f;
  }
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, std::string(f) + ": no device error word");
  const int grid = (int)std::min<int64_t>(p.ntiles, nsm);
  cudaStream_t st = (cudaStream_t)stream;
  if (xt == TQ_F32)
    return alg2 ? launch_tiled_bits<true, true>(p, cb->bits, x, grid, st)
                : launch_tiled_bits<true, false>(p, cb->bits, x, grid, st);
  return alg2 ? launch_tiled_bits<false, true>(p, cb->bits, x, grid, st)
              : launch_tiled_bits<false, false>(p, cb->bits, x, grid, st);
}

}  // namespace tq
