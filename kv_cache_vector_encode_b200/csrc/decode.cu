// Fused TurboQuant decode for d <= 128 (tq_decode):
//   x_hat = n (Pi^T c[idx] + alpha gamma S^T (2z - 1)),  alpha = sqrt(pi/2)/d,
// the second term for Algorithm 2 codes only (ai-navigate-news page: inverse rotation after the
// scalar codebook; Algorithm 2's residual sign term with its norm).
//
// Same transposed orientation as the encoder: D[j][v] = sum_i A[j][i] B[v][i] with A = Pi^T (and
// S^T) resident in shared memory and B = the dequantised tile: B_c[v][i] = c[idx_v,i] split as
// c_hi + 2^-12 c_lo, B_s[v][i] = +-1 (exact). TMEM lane j then holds output coordinate j of every
// vector, so an epilogue warp writes 32 consecutive floats of a row per store.
//   D1a = PiT_hi c_hi,  D1b = PiT_lo c_hi + PiT_hi c_lo,  D2a = ST_hi s,  D2b = ST_lo s
//   x_hat = n ((D1a + 2^-12 D1b) + alpha gamma (D2a + 2^-12 D2b))
// Roles (10 warps): warp 1 owns TMEM and issues MMAs; warps 2-5 load the packed tile and write the
// B operands; warps 6-9 are the epilogue. All waits are bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kDecThreads = 320;

struct DecodeParams {
  int64_t n;
  int d, G, bits, KP, ntiles, dp;
  const __half* pit_hi;
  const __half* pit_lo;
  const __half* st_hi;
  const __half* st_lo;
  const uint32_t* codes;
  const uint32_t* signs;
  const uint16_t* norms;
  const uint16_t* gammas;
  void* out;
  float alpha;
  uint16_t c_hi[16], c_lo[16];
  uint32_t* err;
};

struct DecLayout {
  uint32_t a_bytes, b_bytes;
  uint32_t off_a[4], off_b[3], off_codes, off_signs, off_info, off_bar, total;
};

__host__ __device__ inline uint32_t dround(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <bool ALG2>
__host__ __device__ inline DecLayout dec_layout(int KP, int NV, int G, int bits) {
  DecLayout L{};
  L.a_bytes = 128u * KP * 2;
  L.b_bytes = (uint32_t)NV * KP * 2;
  uint32_t off = 0;
  for (int i = 0; i < (ALG2 ? 4 : 2); ++i) { L.off_a[i] = off; off += L.a_bytes; }
  for (int i = 0; i < (ALG2 ? 3 : 2); ++i) { L.off_b[i] = off; off += L.b_bytes; }
  L.off_codes = off; off += dround((uint32_t)NV * G * bits * 4, 128);
  L.off_signs = off; off += dround((uint32_t)NV * G * 4, 128);
  L.off_info = off; off += 2u * 2 * NV * 4;     // [2 buffers][norm, alpha*gamma][NV]
  L.off_bar = dround(off, 8); off = L.off_bar + 16 * 8;
  L.total = off + 1024;
  return L;
}

enum DBars { B_FULL = 0, B_EMPTY = 1, ACC_FULL = 2, ACC_EMPTY = 4, INFO_EMPTY = 6, UNP = 8, DNBARS = 9 };

template <bool ALG2, int NV, bool OUT_BF16>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr uint32_t COLS = ALG2 ? 4 * NV : 2 * NV;
  constexpr uint32_t NCOLS = 2 * COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const DecLayout Lo = dec_layout<ALG2>(p.KP, NV, p.G, p.bits);
  uint64_t* bar = (uint64_t*)(smem + Lo.off_bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + DNBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + DNBARS) + 1;
  float* info = (float*)(smem + Lo.off_info);
  uint32_t* scodes = (uint32_t*)(smem + Lo.off_codes);
  uint32_t* ssigns = (uint32_t*)(smem + Lo.off_signs);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = p.d, KP = p.KP, G = p.G, bits = p.bits;

  {
    const __half* srcs[4] = {p.pit_hi, p.pit_lo, p.st_hi, p.st_lo};
    const int chunks = KP / 8;
#pragma unroll
    for (int m = 0; m < (ALG2 ? 4 : 2); ++m) {
      uint8_t* dst = smem + Lo.off_a[m];
      for (int c = tid; c < 128 * chunks; c += kDecThreads) {
        int r = c / chunks, kc = c % chunks;
        *(uint4*)(dst + sw128_offset(r, kc * 16, 128)) = *(const uint4*)(srcs[m] + (size_t)r * p.dp + kc * 8);
      }
    }
    if (tid == 0) {
      mbar_init(&bar[B_FULL], 128);
      mbar_init(&bar[B_EMPTY], 1);
      mbar_init(&bar[ACC_FULL], 1); mbar_init(&bar[ACC_FULL + 1], 1);
      mbar_init(&bar[ACC_EMPTY], 128); mbar_init(&bar[ACC_EMPTY + 1], 128);
      mbar_init(&bar[INFO_EMPTY], 128); mbar_init(&bar[INFO_EMPTY + 1], 128);
      mbar_init(&bar[UNP], 128);
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

  if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, NV);
      const uint32_t a0 = smem_u32(smem + Lo.off_a[0]), a1 = smem_u32(smem + Lo.off_a[1]);
      const uint32_t a2 = ALG2 ? smem_u32(smem + Lo.off_a[2]) : 0u, a3 = ALG2 ? smem_u32(smem + Lo.off_a[3]) : 0u;
      const uint32_t bch = smem_u32(smem + Lo.off_b[0]), bcl = smem_u32(smem + Lo.off_b[1]);
      const uint32_t bs = ALG2 ? smem_u32(smem + Lo.off_b[2]) : 0u;
      const int ksteps = KP / 16;
      for (int k = 0; k < my_tiles; ++k) {
        const int a = k & 1;
        if (!mbar_wait(&bar[ACC_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        if (!mbar_wait(&bar[B_FULL], k & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        tc_fence_after();
        const uint32_t d1a = tbase + a * COLS, d1b = d1a + NV, d2a = d1a + 2 * NV, d2b = d1a + 3 * NV;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t kb = ks * 32, blk = kb >> 7, inb = kb & 127;
          const uint32_t ao = blk * 128 * 128 + inb, bo = blk * NV * 128 + inb;
          const uint64_t dch = desc_kmajor_sw128(bch + bo);
          mma_f16_ss(d1a, desc_kmajor_sw128(a0 + ao), dch, idesc, ks > 0);
          mma_f16_ss(d1b, desc_kmajor_sw128(a1 + ao), dch, idesc, ks > 0);
          mma_f16_ss(d1b, desc_kmajor_sw128(a0 + ao), desc_kmajor_sw128(bcl + bo), idesc, 1);
          if (ALG2) {
            const uint64_t dsg = desc_kmajor_sw128(bs + bo);
            mma_f16_ss(d2a, desc_kmajor_sw128(a2 + ao), dsg, idesc, ks > 0);
            mma_f16_ss(d2b, desc_kmajor_sw128(a3 + ao), dsg, idesc, ks > 0);
          }
        }
        mma_commit(&bar[B_EMPTY]);
        mma_commit(&bar[ACC_FULL + a]);
      }
    }
  } else if (warp >= 2 && warp < 6) {
    // ---------------- unpackers: codes -> fp16 B operands -----------------------------------------
    const int ut = tid - 64;               // 0..127
    const int q = ut >> 5;                 // group handled by this warp
    const int i = q * 32 + lane;           // coordinate handled by this thread
    __shared__ __half lut_hi[16], lut_lo[16];
    uint32_t unp_uses = 0;
    // bounded group barrier of the 128 unpacker threads
    auto unp_sync = [&]() -> bool {
      mbar_arrive(&bar[UNP]);
      const bool ok = mbar_wait(&bar[UNP], unp_uses & 1, p.err, kDevTimeoutSync, abort_flag);
      ++unp_uses;
      return ok;
    };
    if (ut < 16) {
      lut_hi[ut] = __ushort_as_half(p.c_hi[ut]);
      lut_lo[ut] = __ushort_as_half(p.c_lo[ut]);
    }
    bool ok = unp_sync();
    for (int k = 0; k < my_tiles && ok; ++k) {
      const int a = k & 1;
      const int64_t v0 = ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
      // stage the packed words of the tile (coalesced loads)
      {
        const int nw = rows * G * bits;
        const uint32_t* src = p.codes + v0 * G * bits;
        for (int w = ut; w < nw; w += 128) scodes[w] = __ldg(src + w);
        if (ALG2) {
          const int ns = rows * G;
          const uint32_t* ss = p.signs + v0 * G;
          for (int w = ut; w < ns; w += 128) ssigns[w] = __ldg(ss + w);
        }
      }
      if (!mbar_wait(&bar[INFO_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      if (ut < NV) {
        float nv = 0.0f, ag = 0.0f;
        if (ut < rows) {
          nv = __half2float(__ushort_as_half(p.norms[v0 + ut]));
          if (ALG2) ag = p.alpha * __half2float(__ushort_as_half(p.gammas[v0 + ut]));
        }
        info[(a * 2 + 0) * NV + ut] = nv;
        info[(a * 2 + 1) * NV + ut] = ag;
      }
      if (!unp_sync()) break;   // staged words visible to all unpackers
      if (!mbar_wait(&bar[B_EMPTY], (k & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      uint8_t* bch = smem + Lo.off_b[0];
      uint8_t* bcl = smem + Lo.off_b[1];
      uint8_t* bsg = ALG2 ? smem + Lo.off_b[2] : nullptr;
      if (i < KP) {
        for (int v = 0; v < NV; ++v) {
          __half ch = __float2half_rn(0.0f), cl = ch, sg = ch;
          if (v < rows && i < d) {
            const uint32_t* wv = scodes + (v * G + q) * bits;
            int idx = 0;
            for (int pl = 0; pl < bits; ++pl) idx |= ((wv[pl] >> lane) & 1u) << pl;
            ch = lut_hi[idx];
            cl = lut_lo[idx];
            if (ALG2) sg = ((ssigns[v * G + q] >> lane) & 1u) ? __float2half_rn(1.0f) : __float2half_rn(-1.0f);
          }
          const uint32_t off = sw128_offset(v, 2 * i, NV);
          *(__half*)(bch + off) = ch;
          *(__half*)(bcl + off) = cl;
          if (ALG2) *(__half*)(bsg + off) = sg;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&bar[B_FULL]);
      ok = unp_sync();          // staging reused by the next tile
    }
  } else if (warp >= 6) {
    // ---------------- epilogue ----------------------------------------------------------------------
    const int q = warp & 3;
    const int j = q * 32 + lane;          // output coordinate
    const bool active = j < d;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    for (int k = 0; k < my_tiles; ++k) {
      const int a = k & 1;
      const int64_t v0 = ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
      if (!mbar_wait(&bar[ACC_FULL + a], (k >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      const uint32_t d1a = tbase + lane_base + a * COLS, d1b = d1a + NV, d2a = d1a + 2 * NV, d2b = d1a + 3 * NV;
      for (int c0 = 0; c0 < NV; c0 += 16) {
        uint32_t ra[16], rb[16], rc[16], rd[16];
        tmem_ld16(d1a + c0, ra);
        tmem_ld16(d1b + c0, rb);
        if (ALG2) {
          tmem_ld16(d2a + c0, rc);
          tmem_ld16(d2b + c0, rd);
        }
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int v = c0 + jj;
          const float nv = info[(a * 2 + 0) * NV + v];
          float val = fmaf(__uint_as_float(rb[jj]), kSplitScaleInv, __uint_as_float(ra[jj]));
          if (ALG2) {
            const float ag = info[(a * 2 + 1) * NV + v];
            const float sv = fmaf(__uint_as_float(rd[jj]), kSplitScaleInv, __uint_as_float(rc[jj]));
            val = fmaf(ag, sv, val);
          }
          val *= nv;
          if (active && v < rows) {
            if (OUT_BF16)
              ((__nv_bfloat16*)p.out)[(v0 + v) * d + j] = __float2bfloat16_rn(val);
            else
              ((float*)p.out)[(v0 + v) * d + j] = val;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[ACC_EMPTY + a]);
      mbar_arrive(&bar[INFO_EMPTY + a]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, NCOLS);
  }
}

template <bool ALG2, int NV, bool BF16>
tq_status launch_decode(DecodeParams& p, cudaStream_t st) {
  const DecLayout Lo = dec_layout<ALG2>(p.KP, NV, p.G, p.bits);
  auto kern = decode_kernel<ALG2, NV, BF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode: shared memory attribute");
  p.ntiles = (int)((p.n + NV - 1) / NV);
  const int grid = std::min(p.ntiles, sm_count());
  kern<<<grid, kDecThreads, Lo.total, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tq_decode: launch");
  return TQ_OK;
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" TQ_API tq_status tq_decode(const tq_codebook* cb, int64_t n, int32_t d, const void* rot, const uint32_t* codes,
                               const uint32_t* signs, const uint16_t* norms, const uint16_t* gammas, void* out,
                               int32_t out_dtype, void* stream) {
  clear_error();
  if (!cb || !rot || !codes || !norms || !out) return fail(TQ_ERR_INVALID_ARG, "tq_decode: NULL pointer");
  if ((signs == nullptr) != (gammas == nullptr))
    return fail(TQ_ERR_INVALID_ARG, "tq_decode: signs and gammas must both be NULL or both be set");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "tq_decode: n < 0");
  if (!valid_dim(d)) return fail(TQ_ERR_UNSUPPORTED, "tq_decode: d must be a multiple of 32 in [32, 4096]");
  if (cb->d != d || cb->bits < 1 || cb->bits > 4 || cb->levels != (1 << cb->bits))
    return fail(TQ_ERR_INVALID_ARG, "tq_decode: codebook does not match d / has bad bits");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "tq_decode: out_dtype");
  if (!aligned16(rot) || !aligned16(codes) || !aligned16(norms) || !aligned16(out) ||
      (signs && (!aligned16(signs) || !aligned16(gammas))))
    return fail(TQ_ERR_INVALID_ARG, "tq_decode: pointers must be 16-byte aligned");
  if (n == 0) return TQ_OK;
  if (d > 128) return fail(TQ_ERR_UNSUPPORTED, "tq_decode: d > 128 is not supported by this build");
  RotLayout RL = rot_layout(d);
  const char* base = (const char*)rot;
  DecodeParams p{};
  p.n = n;
  p.d = d;
  p.G = d / 32;
  p.bits = cb->bits;
  p.KP = d <= 64 ? 64 : 128;
  p.dp = RL.dp;
  p.pit_hi = (const __half*)(base + RL.pit_hi);
  p.pit_lo = (const __half*)(base + RL.pit_lo);
  p.st_hi = (const __half*)(base + RL.st_hi);
  p.st_lo = (const __half*)(base + RL.st_lo);
  p.codes = codes;
  p.signs = signs;
  p.norms = norms;
  p.gammas = gammas;
  p.out = out;
  p.alpha = (float)(std::sqrt(M_PI / 2.0) / d);
  for (int k = 0; k < 16; ++k) {
    float c = k < cb->levels ? cb->c[k] : 0.0f;
    __half h = __float2half_rn(c);
    __half l = __float2half_rn((c - __half2float(h)) * kSplitScale);
    p.c_hi[k] = __half_as_ushort(h);
    p.c_lo[k] = __half_as_ushort(l);
  }
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, "tq_decode: no device error word (is a CUDA device present?)");
  cudaStream_t st = (cudaStream_t)stream;
  const bool bf = out_dtype == TQ_BF16;
  if (signs) return bf ? launch_decode<true, 64, true>(p, st) : launch_decode<true, 64, false>(p, st);
  return bf ? launch_decode<false, 128, true>(p, st) : launch_decode<false, 128, false>(p, st);
}
