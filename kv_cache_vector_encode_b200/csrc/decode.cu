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
// Roles (14 warps): warp 0 bulk-copies the resident operands; warp 1 owns TMEM and issues MMAs;
// warps 2-5 unpack (one thread per (vector, 32-coordinate group), 16-byte swizzled stores into a
// double-buffered operand);
// warps 6-13 are the epilogue (two warps per TMEM lane quarter). All waits are bounded.
//
// Unpacking: for s = 0..3 the nibbles of ((w0 >> s) & 0x11111111) | ((w1 >> s) & 0x11111111) << 1
// | ... are the code indices of coordinates s + 4 n (n = 0..7) of a 32-coordinate group. Used as
// byte-permute selectors over the low and the high bytes of the fp16 levels (up to eight levels;
// sixteen-level codebooks look up the magnitude of the symmetric codebook and flip the sign), four
// coordinates cost two lookups and two interleaves per fp16 part. The group's K order is therefore
// k = 8 s + 4 half + n for coordinate 16 half + 4 n + s, and the resident Pi^T / S^T images (made
// by tq_rotation_prepare for this kernel only) store their K columns in that order.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kDecThreads = 448;

struct DecodeParams {
  int64_t n;
  int d, G, KP, ntiles;
  const uint8_t* img[4];     // PiT_hi, PiT_lo, ST_hi, ST_lo shared-memory images (band 0)
  uint32_t img_bytes;
  const uint32_t* codes;
  const uint32_t* signs;
  const uint16_t* norms;
  const uint16_t* gammas;
  void* out;
  float alpha;
  uint32_t tab[8];                 // level bytes: [0,1] low / [2,3] high bytes of c_hi, [4,5] / [6,7] of c_lo
  // mixed widths per channel group (BITS == 0): group g's width, its first word in the record, the
  // record's words, and the level tables of the codebooks of 1..4 bits
  int gbits[4], goff[4], wv;
  uint32_t tabs[4][8];
  uint32_t* err;
};

struct DecLayout {
  uint32_t a_bytes, b_bytes;
  uint32_t off_a[4], off_b[3], b_set, off_info, off_bar, total;   // buffer s of B plane i: off_b[i] + s * b_set
};

__host__ __device__ inline uint32_t dround(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

template <bool ALG2>
__host__ __device__ inline DecLayout dec_layout(int KP, int NV) {
  DecLayout L{};
  L.a_bytes = 128u * KP * 2;
  L.b_bytes = (uint32_t)NV * KP * 2;
  uint32_t off = 0;
  for (int i = 0; i < (ALG2 ? 4 : 2); ++i) { L.off_a[i] = off; off += L.a_bytes; }
  for (int i = 0; i < (ALG2 ? 3 : 2); ++i) { L.off_b[i] = off; off += L.b_bytes; }
  L.b_set = (ALG2 ? 3 : 2) * L.b_bytes;
  off += L.b_set;
  L.off_info = off; off += 2u * 2 * NV * 4;     // [2 buffers][norm, alpha*gamma][NV]
  L.off_bar = dround(off, 8); off = L.off_bar + 16 * 8;
  L.total = off + 1024;
  return L;
}

enum DBars { A_FULL = 0, B_FULL = 1, B_EMPTY = 3, ACC_FULL = 5, ACC_EMPTY = 7, INFO_EMPTY = 9, DNBARS = 11 };

template <bool ALG2, int NV, bool OUT_BF16, int BITS>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr bool MIX = BITS == 0;          // widths per channel group (Algorithm 1 codes)
  constexpr int BMAX = MIX ? 4 : BITS;
  static_assert(!(MIX && ALG2), "mixed widths are an Algorithm 1 format");
  constexpr uint32_t COLS = ALG2 ? 4 * NV : 2 * NV;
  constexpr uint32_t NCOLS = 2 * COLS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const DecLayout Lo = dec_layout<ALG2>(p.KP, NV);
  uint64_t* bar = (uint64_t*)(smem + Lo.off_bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + DNBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + DNBARS) + 1;
  float* info = (float*)(smem + Lo.off_info);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = p.d, KP = p.KP, G = p.G;
  constexpr int na = ALG2 ? 4 : 2;

  if (tid == 0) {
    mbar_init(&bar[A_FULL], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_FULL + s], 4);          // one arrival per unpacker warp
      mbar_init(&bar[B_EMPTY + s], 1);
      mbar_init(&bar[ACC_FULL + s], 1);
      mbar_init(&bar[ACC_EMPTY + s], 8);       // one arrival per epilogue warp
      mbar_init(&bar[INFO_EMPTY + s], 8);
    }
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

  if (warp == 0) {
    if (elect_one_sync()) {
      mbar_arrive_expect_tx(&bar[A_FULL], na * p.img_bytes);
      for (int m = 0; m < na; ++m) bulk_g2s(smem + Lo.off_a[m], p.img[m], p.img_bytes, &bar[A_FULL]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // warp-uniform schedule (descriptors stay in uniform registers); one elected lane issues
    if (mbar_wait_warp(&bar[A_FULL], 0, p.err, kDevTimeoutLoad, abort_flag)) {
      const uint32_t idesc = idesc_f16_f32(128, NV);
      const uint32_t a0 = smem_u32(smem + Lo.off_a[0]), a1 = smem_u32(smem + Lo.off_a[1]);
      const uint32_t a2 = ALG2 ? smem_u32(smem + Lo.off_a[2]) : 0u, a3 = ALG2 ? smem_u32(smem + Lo.off_a[3]) : 0u;

      const int ksteps = KP / 16;
      for (int k = 0; k < my_tiles; ++k) {
        const int a = k & 1;
        if (!mbar_wait_warp(&bar[ACC_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        if (!mbar_wait_warp(&bar[B_FULL + a], (k >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        tc_fence_after();
        const uint32_t bch = smem_u32(smem + Lo.off_b[0] + a * Lo.b_set), bcl = bch + Lo.b_bytes;
        const uint32_t bs = ALG2 ? bch + 2 * Lo.b_bytes : 0u;
        const uint32_t d1a = tbase + a * COLS, d1b = d1a + NV, d2a = d1a + 2 * NV, d2b = d1a + 3 * NV;
        if (elect_one_sync()) {
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
          mma_commit(&bar[B_EMPTY + a]);
          mma_commit(&bar[ACC_FULL + a]);
        }
        __syncwarp();
      }
    }
  } else if (warp < 6) {
    // ---------------- unpackers: codes -> fp16 B operands -----------------------------------------
    const int ut = tid - 64;               // 0..127
    uint32_t tab[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) tab[k] = p.tab[k];
    const int gp = KP / 32;                  // groups per operand row (padding groups included)
    const int units = NV * gp;
    constexpr int UPT = NV * 4 / 128;        // units per thread (gp <= 4)
    // The code words of a tile are fetched one tile ahead, all loads of a tile issued together,
    // so the unpack does not wait on one global load after another.
    uint32_t cw[UPT][BMAX], cs[UPT];
    uint16_t cn = 0, cg = 0;
    auto fetch = [&](int k, uint32_t (&W)[UPT][BMAX], uint32_t (&SGW)[UPT], uint16_t& nn, uint16_t& gg) {
      const int64_t v0 = ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
#pragma unroll
      for (int j = 0; j < UPT; ++j) {
        const int u = ut + 128 * j, v = u / gp, g = u % gp;
        const bool live = u < units && v < rows && g < G;
        const int gb = MIX ? p.gbits[g < G ? g : 0] : BITS;
        const int64_t wbase = MIX ? (v0 + v) * p.wv + p.goff[g < G ? g : 0] : ((v0 + v) * G + g) * BITS;
#pragma unroll
        for (int pl = 0; pl < BMAX; ++pl) W[j][pl] = (live && pl < gb) ? __ldg(p.codes + wbase + pl) : 0u;
        SGW[j] = (ALG2 && live) ? __ldg(p.signs + (v0 + v) * G + g) : 0u;
      }
      nn = gg = 0;
      if (ut < rows) {
        nn = __ldg(p.norms + v0 + ut);
        if (ALG2) gg = __ldg(p.gammas + v0 + ut);
      }
    };
    if (my_tiles > 0) fetch(0, cw, cs, cn, cg);
    for (int k = 0; k < my_tiles; ++k) {
      const int a = k & 1;
      const int64_t v0 = ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
      uint32_t nw[UPT][BMAX], ns[UPT];
      uint16_t nn = 0, ngm = 0;
      if (k + 1 < my_tiles) fetch(k + 1, nw, ns, nn, ngm);
      if (!mbar_wait_warp(&bar[INFO_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      if (ut < NV) {
        info[(a * 2 + 0) * NV + ut] = __half2float(__ushort_as_half(cn));
        info[(a * 2 + 1) * NV + ut] = ALG2 ? p.alpha * __half2float(__ushort_as_half(cg)) : 0.0f;
      }
      if (!mbar_wait_warp(&bar[B_EMPTY + a], ((k >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
      uint8_t* bch = smem + Lo.off_b[0] + a * Lo.b_set;
      uint8_t* bcl = bch + Lo.b_bytes;
      uint8_t* bsg = ALG2 ? bch + 2 * Lo.b_bytes : nullptr;
#pragma unroll
      for (int j = 0; j < UPT; ++j) {
        const int u = ut + 128 * j;
        if (u >= units) break;
        const int v = u / gp, g = u % gp;
        const bool live = v < rows && g < G;
        const uint32_t* w = cw[j];
        const uint32_t sg = cs[j];
        // this unit's width and level table (a group's own codebook in the mixed format)
        const int gb = MIX ? p.gbits[g < G ? g : 0] : BITS;
        if (MIX) {
#pragma unroll
          for (int t8 = 0; t8 < 8; ++t8) tab[t8] = p.tabs[gb - 1][t8];
        }
        // selector planes: the index bits (up to 3), or for 16 levels the magnitude bits
        // (low bits ^ ~top bit) with the sign taken from the top bit
        const int SB = gb < 4 ? gb : 3;
        const uint32_t flip = gb == 4 ? ~w[BMAX == 4 ? 3 : 0] : 0u;
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          uint32_t x = 0;
#pragma unroll
          for (int pl = 0; pl < (BMAX < 4 ? BMAX : 3); ++pl)
            if (pl < SB) x |= (((w[pl] ^ flip) >> s4) & 0x11111111u) << pl;
          const uint32_t fl = gb == 4 ? (flip >> s4) & 0x11111111u : 0u;
          uint32_t o_hi[4], o_lo[4], o_s[4];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t sel = half ? x >> 16 : x;
            uint32_t hb = __byte_perm(tab[2], tab[3], sel), hl = __byte_perm(tab[6], tab[7], sel);
            if (gb == 4) {
              const uint32_t sb = __byte_perm(0x8000u, 0u, half ? fl >> 16 : fl);   // 0x80 where negative
              hb ^= sb;
              hl ^= sb;
            }
            const uint32_t lb = __byte_perm(tab[0], tab[1], sel), ll = __byte_perm(tab[4], tab[5], sel);
            o_hi[2 * half] = live ? __byte_perm(lb, hb, 0x5140u) : 0u;
            o_hi[2 * half + 1] = live ? __byte_perm(lb, hb, 0x7362u) : 0u;
            o_lo[2 * half] = live ? __byte_perm(ll, hl, 0x5140u) : 0u;
            o_lo[2 * half + 1] = live ? __byte_perm(ll, hl, 0x7362u) : 0u;
            if (ALG2) {
              // z = 1 -> +1 (0x3C00), z = 0 -> -1 (0xBC00)
              const uint32_t zs = ((~sg >> s4) & 0x11111111u) >> (half ? 16 : 0);
              const uint32_t zb = __byte_perm(0xBC3Cu, 0u, zs);
              o_s[2 * half] = live ? __byte_perm(0u, zb, 0x5140u) : 0u;
              o_s[2 * half + 1] = live ? __byte_perm(0u, zb, 0x7362u) : 0u;
            }
          }
          const uint32_t off = sw128_offset(v, (g * 32 + s4 * 8) * 2, NV);
          *(uint4*)(bch + off) = make_uint4(o_hi[0], o_hi[1], o_hi[2], o_hi[3]);
          *(uint4*)(bcl + off) = make_uint4(o_lo[0], o_lo[1], o_lo[2], o_lo[3]);
          if (ALG2) *(uint4*)(bsg + off) = make_uint4(o_s[0], o_s[1], o_s[2], o_s[3]);
        }
      }
#pragma unroll
      for (int j = 0; j < UPT; ++j) {
#pragma unroll
        for (int pl = 0; pl < BMAX; ++pl) cw[j][pl] = nw[j][pl];
        cs[j] = ns[j];
      }
      cn = nn;
      cg = ngm;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_FULL + a]);
    }
  } else {
    // ---------------- epilogue ----------------------------------------------------------------------
    const int e = warp - 6;
    const int q = warp & 3;
    const int j = q * 32 + lane;          // output coordinate
    const bool active = j < d;
    const int cbeg = (e >> 2) * (NV / 2), cend = cbeg + NV / 2;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    for (int k = 0; k < my_tiles; ++k) {
      const int a = k & 1;
      const int64_t v0 = ((int64_t)blockIdx.x + (int64_t)k * gridDim.x) * NV;
      const int rows = (int)min((int64_t)NV, p.n - v0);
      if (!mbar_wait_warp(&bar[ACC_FULL + a], (k >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      const uint32_t d1a = tbase + lane_base + a * COLS, d1b = d1a + NV, d2a = d1a + 2 * NV, d2b = d1a + 3 * NV;
      for (int c0 = cbeg; c0 < cend; c0 += 16) {
        uint32_t ra[16], rb[16], rc[16], rd[16];
        tmem_ld16(d1a + c0, ra);
        tmem_ld16(d1b + c0, rb);
        if (ALG2) {
          tmem_ld16(d2a + c0, rc);
          tmem_ld16(d2b + c0, rd);
        }
        // Algorithm 1: the 16 vectors' norms as four 16-byte loads (Algorithm 2 reads its scales one
        // by one, which keeps its four TMEM blocks in registers)
        float nvs[16];
        if (!ALG2) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float4 f = *(const float4*)&info[(a * 2 + 0) * NV + c0 + 4 * u];
            nvs[4 * u] = f.x;
            nvs[4 * u + 1] = f.y;
            nvs[4 * u + 2] = f.z;
            nvs[4 * u + 3] = f.w;
          }
        }
        tmem_ld_wait();
        // row pointers advance by d elements per vector; a full batch needs no row check
        const bool full = c0 + 16 <= rows;
        const size_t row0 = (size_t)(v0 + c0) * d + j;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          float val = fmaf(__uint_as_float(rb[jj]), kSplitScaleInv, __uint_as_float(ra[jj]));
          if (ALG2) {
            const float sv = fmaf(__uint_as_float(rd[jj]), kSplitScaleInv, __uint_as_float(rc[jj]));
            val = fmaf(info[(a * 2 + 1) * NV + c0 + jj], sv, val);
          }
          val *= ALG2 ? info[(a * 2 + 0) * NV + c0 + jj] : nvs[jj];
          if (active && (full || c0 + jj < rows)) {
            const size_t o = row0 + (size_t)jj * d;
            if (OUT_BF16)
              ((__nv_bfloat16*)p.out)[o] = __float2bfloat16_rn(val);
            else
              ((float*)p.out)[o] = val;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[ACC_EMPTY + a]);
        mbar_arrive(&bar[INFO_EMPTY + a]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, NCOLS);
  }
}

template <bool ALG2, int NV, bool BF16, int BITS>
tq_status launch_decode(DecodeParams& p, cudaStream_t st) {
  const DecLayout Lo = dec_layout<ALG2>(p.KP, NV);
  auto kern = decode_kernel<ALG2, NV, BF16, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode: shared memory attribute");
  p.ntiles = (int)((p.n + NV - 1) / NV);
  const int grid = std::min(p.ntiles, sm_count());
  kern<<<grid, kDecThreads, Lo.total, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tq_decode: launch");
  return TQ_OK;
}

// Byte tables of the fp16 hi / lo parts of a codebook's levels for the byte-permute lookup: up to
// eight levels are looked up directly; sixteen by magnitude (the positive half c[8 + m]).
void level_tables(const tq_codebook* cb, uint32_t (&tab)[8]) {
  const int L = cb->levels;
  const int base_level = L > 8 ? L / 2 : 0, nt = L > 8 ? 8 : L;
  uint8_t hl[4][8] = {};                       // [low c_hi, high c_hi, low c_lo, high c_lo][entry]
  for (int m = 0; m < nt; ++m) {
    const float c = cb->c[base_level + m];
    const __half h = __float2half_rn(c);
    const __half l = __float2half_rn((c - __half2float(h)) * kSplitScale);
    const uint16_t hu = __half_as_ushort(h), lu = __half_as_ushort(l);
    hl[0][m] = (uint8_t)(hu & 0xFF);
    hl[1][m] = (uint8_t)(hu >> 8);
    hl[2][m] = (uint8_t)(lu & 0xFF);
    hl[3][m] = (uint8_t)(lu >> 8);
  }
  for (int t = 0; t < 4; ++t)
    for (int w = 0; w < 2; ++w)
      tab[2 * t + w] = (uint32_t)hl[t][4 * w] | (uint32_t)hl[t][4 * w + 1] << 8 | (uint32_t)hl[t][4 * w + 2] << 16 |
                       (uint32_t)hl[t][4 * w + 3] << 24;
}

template <bool ALG2, int NV, bool BF16>
tq_status decode_bits(DecodeParams& p, int bits, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_decode<ALG2, NV, BF16, 1>(p, st);
    case 2: return launch_decode<ALG2, NV, BF16, 2>(p, st);
    case 3: return launch_decode<ALG2, NV, BF16, 3>(p, st);
    default: return launch_decode<ALG2, NV, BF16, 4>(p, st);
  }
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" TQ_API tq_status tq_decode(const tq_codebook* cb, int64_t n, int32_t d, const void* rot,
                                      const uint32_t* codes, const uint32_t* signs, const uint16_t* norms,
                                      const uint16_t* gammas, void* out, int32_t out_dtype, void* stream) {
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
  const uint8_t* base = (const uint8_t*)rot;
  DecodeParams p{};
  p.n = n;
  p.d = d;
  p.G = d / 32;
  p.KP = d <= 64 ? 64 : 128;
  p.img[0] = base + RL.pit_hi;
  p.img[1] = base + RL.pit_lo;
  p.img[2] = base + RL.st_hi;
  p.img[3] = base + RL.st_lo;
  p.img_bytes = 128u * p.KP * 2;
  p.codes = codes;
  p.signs = signs;
  p.norms = norms;
  p.gammas = gammas;
  p.out = out;
  p.alpha = (float)(std::sqrt(M_PI / 2.0) / d);
  const int L = cb->levels;
  for (int k = 0; k < L; ++k)
    if (cb->c[L - 1 - k] != -cb->c[k]) return fail(TQ_ERR_INVALID_ARG, "tq_decode: codebook is not symmetric");
  level_tables(cb, p.tab);
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, "tq_decode: no device error word (is a CUDA device present?)");
  cudaStream_t st = (cudaStream_t)stream;
  const bool bf = out_dtype == TQ_BF16;
  if (signs) return bf ? decode_bits<true, 64, true>(p, cb->bits, st) : decode_bits<true, 64, false>(p, cb->bits, st);
  return bf ? decode_bits<false, 128, true>(p, cb->bits, st) : decode_bits<false, 128, false>(p, cb->bits, st);
}

// Decode of the mixed-width format of tq_encode_mse_mixed (d <= 128): each unpacking thread expands
// its (vector, group) unit with the group's own codebook.
extern "C" TQ_API tq_status tq_decode_mixed(const tq_codebook* cbs, const int32_t* group_bits, int64_t n, int32_t d,
                                            const void* rot, const uint32_t* codes, const uint16_t* norms, void* out,
                                            int32_t out_dtype, void* stream) {
  clear_error();
  const char* f = "tq_decode_mixed";
  if (!cbs || !group_bits || !rot || !codes || !norms || !out) return fail(TQ_ERR_INVALID_ARG, "tq_decode_mixed: NULL pointer");
  if (n < 0) return fail(TQ_ERR_INVALID_ARG, "tq_decode_mixed: n < 0");
  if (!valid_dim(d) || d > 128) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_mixed: d must be 32, 64, 96 or 128");
  if (out_dtype != TQ_F32 && out_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_mixed: out_dtype");
  DecodeParams p{};
  const int G = d / 32;
  int wv = 0;
  for (int g = 0; g < G; ++g) {
    const int b = group_bits[g];
    if (b < 1 || b > 4) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_mixed: group widths must be 1..4 bits");
    const tq_codebook* cb = &cbs[b - 1];
    if (cb->d != d || cb->bits != b || cb->levels != (1 << b))
      return fail(TQ_ERR_INVALID_ARG, "tq_decode_mixed: cbs[b - 1] must be the b-bit codebook for this d");
    const int L = cb->levels;
    for (int k = 0; k < L; ++k)
      if (cb->c[L - 1 - k] != -cb->c[k]) return fail(TQ_ERR_INVALID_ARG, "tq_decode_mixed: codebook is not symmetric");
    p.gbits[g] = b;
    p.goff[g] = wv;
    wv += b;
    level_tables(cb, p.tabs[b - 1]);
  }
  p.wv = wv;
  if (!aligned16(rot) || !aligned16(codes) || !aligned16(norms) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "tq_decode_mixed: pointers must be 16-byte aligned");
  if (n == 0) return TQ_OK;
  RotLayout RL = rot_layout(d);
  const uint8_t* base = (const uint8_t*)rot;
  p.n = n;
  p.d = d;
  p.G = G;
  p.KP = d <= 64 ? 64 : 128;
  p.img[0] = base + RL.pit_hi;
  p.img[1] = base + RL.pit_lo;
  p.img[2] = base + RL.st_hi;
  p.img[3] = base + RL.st_lo;
  p.img_bytes = 128u * p.KP * 2;
  p.codes = codes;
  p.norms = norms;
  p.out = out;
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, std::string(f) + ": no device error word");
  cudaStream_t st = (cudaStream_t)stream;
  return out_dtype == TQ_BF16 ? launch_decode<false, 128, true, 0>(p, st) : launch_decode<false, 128, false, 0>(p, st);
}
