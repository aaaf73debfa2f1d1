// Decode attention over a TurboQuant-packed KV cache (tq_attend_decode).
//
// Method (aiboss88 page: attention evaluated on the quantised cache, unbiased inner-product
// estimates; ai-navigate-news page: keys by Algorithm 1, values by Algorithm 2):
//   out[b][h] = sum_t softmax_t(scale <q, k_hat_t>) v_hat_t,   k_hat_t = n_t Pi^T c_K[idx_t],
//   v_hat_t = m_t (Pi^T c_V[jdx_t] + alpha gamma_t S^T (2 z_t - 1)).
// Evaluated from the codes, never materialising k_hat or v_hat:
//   * the query is rotated once, q' = Pi q (prep kernel);
//   * the codebook is an odd function of the index bits (exact symmetry), so c[idx] =
//     sum_S beta_S prod_{p in S} (1 - 2 bit_p) over the odd subsets S of the bit planes
//     (Walsh expansion). With b_S = XOR of the planes in S,
//       <q', c[idx]> = sum_S beta_S (Q - 2 <q', b_S>),   Q = sum_i q'_i,
//     and <q', b_S> is an exact integer tensor-core product: A = the bits b_S (0/1 bytes, scaled
//     by 2^s, see below), B = beta_S q' in 32-bit fixed point as four signed 8-bit limbs;
//   * values are accumulated in the rotated / sign domain: for each V plane P (the Walsh
//     planes of the value codes and the sign plane), Y_P[i] = sum_t w_t b_P,t,i with the softmax
//     weights w_t (times the value norm, times gamma for the sign plane) in 32-bit unsigned fixed
//     point as four 8-bit limbs; then o_rot = sum_S beta_S (W - 2 Y_S), o_sign = 2 Y_z - W'
//     (W = sum_t w_t) and, once per query head, out = Pi^T o_rot / l + alpha S^T o_sign / l.
//
// Bit expansion: a 32-bit plane word w covers 32 coordinates; register s (s = 0..7) of
// (w & (0x01010101 << s)) holds coordinates s, 8+s, 16+s, 24+s as bytes 0 or 2^s. The tensor-core
// index order inside each 32-coordinate group is therefore k = 4 s + j for coordinate 8 j + s,
// and the 2^s factor is divided out of the query limbs (scores) or of the output rows (values).
//
// Kernels: prep (q' limbs, per-head constants), main (persistent; one CTA per SM walks a
// contiguous range of 128-token chunks, possibly spanning several (batch, KV head) slices), combine
// (merges the per-CTA partial softmax states of a slice and applies Pi^T, S^T).
// Main-kernel roles (14 warps): 0 bulk-copies packed chunks; 1 owns TMEM and issues the MMAs;
// 2-5 token warps (thread = token: expand K into TMEM, then softmax of the chunk); 6-9 expand V
// into shared memory; 10-13 accumulate the value products (thread = coordinate).
// All waits are bounded (sm100.cuh).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <vector>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kAttThreads = 448;
constexpr int kChunk = 128;                 // tokens per chunk
constexpr int kStages = 4;                  // packed-chunk ring
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------------------------------------
// Parameters shared by the three kernels
// ------------------------------------------------------------------------------------------------
struct AttParams {
  int B, Hq, Hkv, Hg, d, G;
  int64_t T;
  int slices, nchunk, per_cta, maxseg;
  int bk, mk, kmask[4];          // key bits, number of key Walsh planes, plane subsets
  int bv, mv, vmask[4], vsign;   // value codebook bits, value Walsh planes, subsets, sign plane?
  int np;                        // value planes (mv + vsign)
  int nq, nvc;                   // MMA N for scores / values (Hg * 4 rounded up to 16)
  float beta_k[4], beta_v[4];
  float scale_log2e, alpha;
  const void* q;
  int q_bf16;
  const float* Pi;
  const float* S;
  const uint32_t* k_codes;
  const uint16_t* k_norms;
  const uint32_t* v_codes;
  const uint32_t* v_signs;
  const uint16_t* v_norms;
  const uint16_t* v_gammas;
  uint8_t* bq_img;               // [slices][nq rows x mk*d bytes] K-major SW128 image
  float* head_c;                 // [slices][8][2]: 2^-F_h, Q_h * sum beta
  float* partial;                // [slices][maxseg][Hg][4 + 2d]
  float* out;
  uint32_t* err;
};

__host__ __device__ inline int att_rec(int d) { return 4 + 2 * d; }

// ------------------------------------------------------------------------------------------------
// prep: q' = Pi q per query head, fixed-point limbs of beta_S q' (scaled by 2^-s), constants
// ------------------------------------------------------------------------------------------------
__global__ void attend_prep_kernel(const __grid_constant__ AttParams p) {
  const int slice = blockIdx.x;                  // = b * Hkv + hk
  const int b = slice / p.Hkv, hk = slice % p.Hkv;
  const int d = p.d, i = threadIdx.x;            // coordinate (128 threads)
  const int warp = i >> 5, lane = i & 31;
  __shared__ float sq[8][128];
  __shared__ double qr[8][128];
  __shared__ double red[128];
  const int kbytes = p.mk * d;
  uint8_t* img = p.bq_img + (size_t)slice * p.nq * kbytes;
  for (int o = i; o < p.nq * kbytes / 16; o += blockDim.x) ((uint4*)img)[o] = make_uint4(0, 0, 0, 0);
  for (int h = 0; h < p.Hg; ++h) {
    const size_t qoff = ((size_t)b * p.Hq + hk * p.Hg + h) * d;
    sq[h][i] = p.q_bf16 ? __uint_as_float((uint32_t)((const uint16_t*)p.q)[qoff + i] << 16)
                        : ((const float*)p.q)[qoff + i];
  }
  __syncthreads();
  // q'_h = Pi q_h: one warp per output coordinate, lanes across the row of Pi (coalesced)
  for (int r = warp; r < d; r += 4) {
    const float* row = p.Pi + (size_t)r * d;
    double acc[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) acc[h] = 0.0;
    for (int j = lane; j < d; j += 32) {
      const double pij = (double)row[j];
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < p.Hg) acc[h] = fma(pij, (double)sq[h][j], acc[h]);
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < p.Hg) {
        double v = acc[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) qr[h][r] = v;
      }
    }
  }
  __syncthreads();
  double bmax = 0.0, sb = 0.0;
  for (int S = 0; S < p.mk; ++S) {
    bmax = fmax(bmax, fabs((double)p.beta_k[S]));
    sb += (double)p.beta_k[S];
  }
  for (int h = 0; h < p.Hg; ++h) {
    const double qi = qr[h][i];
    red[i] = qi;
    __syncthreads();
    for (int o = 64; o > 0; o >>= 1) {
      if (i < o) red[i] += red[i + o];
      __syncthreads();
    }
    const double Qh = red[0];
    __syncthreads();
    red[i] = fabs(qi) * bmax;
    __syncthreads();
    for (int o = 64; o > 0; o >>= 1) {
      if (i < o) red[i] = fmax(red[i], red[i + o]);
      __syncthreads();
    }
    const double vmax = red[0];
    __syncthreads();
    int F = 0;
    if (vmax > 0.0) {
      int E;
      frexp(vmax, &E);              // vmax < 2^E
      F = 30 - E;                   // vmax * 2^F < 2^30
    }
    if (i == 0) {
      p.head_c[(slice * 8 + h) * 2 + 0] = (float)ldexp(1.0, -F);
      p.head_c[(slice * 8 + h) * 2 + 1] = (float)(Qh * sb);
    }
    const int g = i >> 5, rr = i & 31, jj = rr >> 3, s = rr & 7;   // coordinate 32g + 8jj + s
    const int kin = 32 * g + 4 * s + jj;                          // its k index inside a plane
    for (int S = 0; S < p.mk; ++S) {
      long long v = llrint(ldexp((double)p.beta_k[S] * qi, F - s));
      const int k = S * d + kin;
      for (int l = 0; l < 4; ++l) {
        const long long dl = l < 3 ? (((v + 128) & 255) - 128) : v;   // balanced signed digits
        v = (v - dl) >> 8;
        img[sw128_offset(h * 4 + l, k, p.nq)] = (uint8_t)(int8_t)dl;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// main kernel
// ------------------------------------------------------------------------------------------------
struct AttLayout {
  uint32_t stage_bytes, kc_bytes, vc_bytes;
  uint32_t off_stage, off_av, av_bytes, off_bw, bw_bytes, off_bq, bq_bytes, off_sc, off_red, off_bar, total;
};

__host__ __device__ inline uint32_t aru(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline AttLayout att_layout(const AttParams& p) {
  AttLayout L{};
  L.kc_bytes = kChunk * p.G * p.bk * 4;
  L.vc_bytes = kChunk * p.G * (p.bv + (p.vsign ? 1 : 0)) * 4;
  L.stage_bytes = aru(L.kc_bytes + L.vc_bytes, 1024);
  uint32_t off = 0;
  L.off_stage = off; off += kStages * L.stage_bytes;
  L.av_bytes = kChunk * 128;                       // one plane: 128 tokens x 128 coordinates
  L.off_av = off; off += 2 * p.np * L.av_bytes;
  L.bw_bytes = (p.nvc / 16) * kChunk * 16;         // one kind: nvc/16 blocks of 128 x 16 bytes
  L.off_bw = off; off += 2 * 2 * L.bw_bytes;
  L.bq_bytes = aru(p.nq * p.mk * p.d, 1024);
  L.off_bq = off; off += 2 * L.bq_bytes;
  L.off_sc = off; off += 4 * 64 * 4;               // chunk scalars, 4-deep ring of 64 floats
  L.off_red = off; off += 512 * 4;                 // cross-warp reductions of the token warps
  L.off_bar = aru(off, 8); off = L.off_bar + 64 * 8;
  L.total = off + 1024;
  return L;
}

enum ABars {
  ST_FULL = 0,                       // [kStages]
  ST_EMPTY = ST_FULL + kStages,      // [kStages]  (K and V expanders: 8 warps)
  BQ_FULL = ST_EMPTY + kStages,      // [2]
  BQ_EMPTY = BQ_FULL + 2,            // [2]
  AK_FULL = BQ_EMPTY + 2,            // [2]  token warps -> MMA (4 warps)
  SC_DONE = AK_FULL + 2,             // [2]  scores MMA complete (commit)
  BW_FULL = SC_DONE + 2,             // [2]  token warps -> MMA (4 warps)
  AV_FULL = BW_FULL + 2,             // [2]  V expanders -> MMA (4 warps)
  V_DONE = AV_FULL + 2,              // [2]  value MMA complete (commit)
  DV_EMPTY = V_DONE + 2,             // [2]  accumulators -> MMA (4 warps)
  SCAL_FULL = DV_EMPTY + 2,          // [4]  token warps -> accumulators: chunk scalars (4 warps)
  TOK = SCAL_FULL + 4,               // token-warp group sync (4 warps)
  ANBARS = TOK + 1
};

// TMEM columns
constexpr uint32_t kAK0 = 0;     // [2][128]
constexpr uint32_t kDS0 = 256;   // [2][<=32]
constexpr uint32_t kDV0 = 320;   // [2][np][<=32]

// chunk c of this CTA -> (slice, chunk within slice)
struct ChunkPos {
  int slice, cis;   // cis = chunk index inside the slice
};
__device__ __forceinline__ ChunkPos chunk_pos(const AttParams& p, int gchunk) {
  ChunkPos r;
  r.slice = gchunk / p.nchunk;
  r.cis = gchunk - r.slice * p.nchunk;
  return r;
}

template <int HG>
__global__ void __launch_bounds__(kAttThreads, 1) attend_main_kernel(const __grid_constant__ AttParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const AttLayout Lo = att_layout(p);
  uint64_t* bar = (uint64_t*)(smem + Lo.off_bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + ANBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + ANBARS) + 1;
  float* scal = (float*)(smem + Lo.off_sc);
  float* red = (float*)(smem + Lo.off_red);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = p.slices * p.nchunk;
  const int c_begin = blockIdx.x * p.per_cta;
  const int c_end = min(total, c_begin + p.per_cta);
  const int nmy = max(0, c_end - c_begin);
  const int d = p.d, G = p.G;
  const int64_t T = p.T;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bar[ST_FULL + s], 1);
      mbar_init(&bar[ST_EMPTY + s], 8);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[BQ_FULL + s], 1);
      mbar_init(&bar[BQ_EMPTY + s], 1);
      mbar_init(&bar[AK_FULL + s], 4);
      mbar_init(&bar[SC_DONE + s], 1);
      mbar_init(&bar[BW_FULL + s], 4);
      mbar_init(&bar[AV_FULL + s], 4);
      mbar_init(&bar[V_DONE + s], 1);
      mbar_init(&bar[DV_EMPTY + s], 4);
    }
    for (int s = 0; s < 4; ++s) mbar_init(&bar[SCAL_FULL + s], 4);
    mbar_init(&bar[TOK], 4);
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

  // segment bookkeeping: a new segment starts at the first chunk and whenever the slice changes
  auto seg_index = [&](int c) -> int {     // ordinal of the segment chunk c (0-based, local) belongs to
    const int s0 = chunk_pos(p, c_begin).slice;
    return chunk_pos(p, c_begin + c).slice - s0;
  };
  auto seg_first = [&](int c) -> bool {
    return c == 0 || chunk_pos(p, c_begin + c).cis == 0;
  };
  auto seg_last = [&](int c) -> bool {
    return c == nmy - 1 || chunk_pos(p, c_begin + c).cis == p.nchunk - 1;
  };

  if (warp == 0) {
    // ------------------------------------ producer -------------------------------------------------
    if (lane == 0) {
      for (int c = 0; c < nmy; ++c) {
        const ChunkPos cp = chunk_pos(p, c_begin + c);
        if (seg_first(c)) {
          const int sg = seg_index(c);
          if (!mbar_wait(&bar[BQ_EMPTY + (sg & 1)], ((sg >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
          const uint32_t nb = (uint32_t)(p.nq * p.mk * d);
          mbar_arrive_expect_tx(&bar[BQ_FULL + (sg & 1)], nb);
          bulk_g2s(smem + Lo.off_bq + (sg & 1) * Lo.bq_bytes, p.bq_img + (size_t)cp.slice * nb, nb,
                   &bar[BQ_FULL + (sg & 1)]);
        }
        const int st = c % kStages;
        if (!mbar_wait(&bar[ST_EMPTY + st], ((c / kStages) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        const int64_t t0 = (int64_t)cp.cis * kChunk;
        const int tc = (int)min((int64_t)kChunk, T - t0);
        const int64_t vec0 = (int64_t)cp.slice * T + t0;       // record index of the first token
        const uint32_t kb = (uint32_t)tc * G * p.bk * 4;
        const uint32_t vb = (uint32_t)tc * G * p.bv * 4;
        const uint32_t sb = p.vsign ? (uint32_t)tc * G * 4 : 0u;
        mbar_arrive_expect_tx(&bar[ST_FULL + st], kb + vb + sb);
        uint8_t* stg = smem + Lo.off_stage + st * Lo.stage_bytes;
        bulk_g2s(stg, p.k_codes + vec0 * G * p.bk, kb, &bar[ST_FULL + st]);
        bulk_g2s(stg + Lo.kc_bytes, p.v_codes + vec0 * G * p.bv, vb, &bar[ST_FULL + st]);
        if (p.vsign)
          bulk_g2s(stg + Lo.kc_bytes + kChunk * G * p.bv * 4, p.v_signs + vec0 * G, sb, &bar[ST_FULL + st]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------ MMA issuer -----------------------------------------------
    if (lane == 0) {
      const uint32_t id_s = idesc_i8_s32(128, p.nq, false, true, false, false);
      const uint32_t id_v = idesc_i8_s32(128, p.nvc, false, false, true, true);
      const int ksteps = p.mk * d / 32;
      auto issue_v = [&](int c) -> bool {
        const int b = c & 1;
        if (!mbar_wait(&bar[BW_FULL + b], (c >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) return false;
        if (!mbar_wait(&bar[AV_FULL + b], (c >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) return false;
        if (!mbar_wait(&bar[DV_EMPTY + b], ((c >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) return false;
        tc_fence_after();
        for (int P = 0; P < p.np; ++P) {
          const bool sgn = p.vsign && P == p.np - 1;
          const uint32_t a0 = smem_u32(smem + Lo.off_av + (b * p.np + P) * Lo.av_bytes);
          const uint32_t b0 = smem_u32(smem + Lo.off_bw + (b * 2 + (sgn ? 1 : 0)) * Lo.bw_bytes);
          const uint32_t dcol = tbase + kDV0 + (b * p.np + P) * p.nvc;
          for (int ks = 0; ks < kChunk / 32; ++ks) {
            const uint64_t da = desc_smem(a0 + ks * 32 * 128, 1024, 1024, 2);
            const uint64_t db = desc_smem(b0 + ks * 32 * 16, 128, kChunk * 16, 0);
            mma_i8_ss(dcol, da, db, id_v, ks > 0);
          }
        }
        mma_commit(&bar[V_DONE + b]);
        return true;
      };
      bool ok = true;
      for (int c = 0; c < nmy && ok; ++c) {
        const int b = c & 1;
        const int sg = seg_index(c);
        if (seg_first(c)) {
          if (!mbar_wait(&bar[BQ_FULL + (sg & 1)], (sg >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag)) break;
        }
        if (!mbar_wait(&bar[AK_FULL + b], (c >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        // D_s[b] is free once the token warps finished chunk c-2 (they arrive BW_FULL after reading it)
        if (c >= 2 && !mbar_wait(&bar[BW_FULL + b], ((c - 2) >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
        tc_fence_after();
        const uint32_t bq = smem_u32(smem + Lo.off_bq + (sg & 1) * Lo.bq_bytes);
        const uint32_t ak = tbase + kAK0 + b * 128;
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t kbyte = ks * 32, blk = kbyte >> 7, inb = kbyte & 127;
          mma_i8_ts(tbase + kDS0 + b * 32, ak + ks * 8, desc_kmajor_sw128(bq + blk * p.nq * 128 + inb), id_s, ks > 0);
        }
        mma_commit(&bar[SC_DONE + b]);
        if (seg_last(c)) mma_commit(&bar[BQ_EMPTY + (sg & 1)]);
        if (c >= 1) ok = issue_v(c - 1);
      }
      if (ok && nmy >= 1 && !*abort_flag) issue_v(nmy - 1);
    }
  } else if (warp < 6) {
    // ------------------------------------ token warps ----------------------------------------------
    const int q = warp & 3;
    const int t = q * 32 + lane;                    // token inside the chunk == TMEM lane
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int Hg = p.Hg;
    uint32_t tok_uses = 0;
    auto tok_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[TOK]);
      const bool ok = mbar_wait_warp(&bar[TOK], tok_uses & 1, p.err, kDevTimeoutSync, abort_flag);
      ++tok_uses;
      return ok;
    };
    // expand the key codes of chunk c into TMEM (A operand of the scores MMA)
    auto expand_k = [&](int c) -> bool {
      const int st = c % kStages, b = c & 1;
      if (!mbar_wait_warp(&bar[ST_FULL + st], (c / kStages) & 1, p.err, kDevTimeoutLoad, abort_flag)) return false;
      if (c >= 2 && !mbar_wait_warp(&bar[SC_DONE + b], ((c - 2) >> 1) & 1, p.err, kDevTimeoutMma, abort_flag))
        return false;
      tc_fence_after();
      const ChunkPos cp = chunk_pos(p, c_begin + c);
      const int tc = (int)min((int64_t)kChunk, T - (int64_t)cp.cis * kChunk);
      const bool live = t < tc;
      // the token's G * bk plane words (<= 16, contiguous, 16-byte aligned)
      const uint4* kw4 = (const uint4*)((const uint32_t*)(smem + Lo.off_stage + st * Lo.stage_bytes) + t * 4 * p.bk);
      uint32_t kw[16];
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        uint4 x = make_uint4(0, 0, 0, 0);
        if (v4 < p.bk && live) x = kw4[v4];
        kw[4 * v4] = x.x;
        kw[4 * v4 + 1] = x.y;
        kw[4 * v4 + 2] = x.z;
        kw[4 * v4 + 3] = x.w;
      }
      const uint32_t ak = tbase + lane_base + kAK0 + b * 128;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t pw[4];
#pragma unroll
        for (int pl = 0; pl < 4; ++pl) {
          // word (g, pl) of a bk-plane record sits at g * bk + pl; bk is 1..3 (selects keep kw in registers)
          const uint32_t w3 = pl < 3 ? kw[3 * g + (pl < 3 ? pl : 0)] : 0u;
          const uint32_t w2 = pl < 2 ? kw[2 * g + (pl < 2 ? pl : 0)] : 0u;
          const uint32_t w1 = pl < 1 ? kw[g] : 0u;
          pw[pl] = p.bk == 3 ? w3 : (p.bk == 2 ? w2 : w1);
        }
#pragma unroll
        for (int S = 0; S < 4; ++S) {
          if (S < p.mk) {
            const int m = p.kmask[S];
            const uint32_t w = ((m & 1) ? pw[0] : 0u) ^ ((m & 2) ? pw[1] : 0u) ^ ((m & 4) ? pw[2] : 0u);
            uint32_t r[8];
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) r[s8] = w & (0x01010101u << s8);
            tmem_st8(ak + S * 32 + g * 8, r);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[AK_FULL + b]);
        mbar_arrive(&bar[ST_EMPTY + st]);
      }
      return true;
    };
    float m2run[HG];   // running max (log2 domain), kept by every thread
    bool ok = nmy > 0 ? expand_k(0) : true;
    for (int c = 0; c < nmy && ok; ++c) {
      const int b = c & 1;
      const ChunkPos cp = chunk_pos(p, c_begin + c);
      const int64_t t0 = (int64_t)cp.cis * kChunk;
      const int tc = (int)min((int64_t)kChunk, T - t0);
      const bool live = t < tc;
      if (seg_first(c)) {
#pragma unroll
        for (int h = 0; h < HG; ++h) m2run[h] = -INFINITY;
      }
      // per-token inputs (plain loads, issued before the waits)
      const int64_t rec = (int64_t)cp.slice * T + t0 + t;
      const float nk = live ? __half2float(__ushort_as_half(__ldg(p.k_norms + rec))) : 0.0f;
      const float nv = live ? __half2float(__ushort_as_half(__ldg(p.v_norms + rec))) : 0.0f;
      const float gm = (live && p.vsign) ? __half2float(__ushort_as_half(__ldg(p.v_gammas + rec))) : 0.0f;
      const float4* hc4 = (const float4*)(p.head_c + cp.slice * 16);
      float hcf[2 * HG];
#pragma unroll
      for (int h2 = 0; h2 < HG / 2; ++h2) {
        const float4 x = __ldg(hc4 + h2);
        hcf[4 * h2] = x.x;
        hcf[4 * h2 + 1] = x.y;
        hcf[4 * h2 + 2] = x.z;
        hcf[4 * h2 + 3] = x.w;
      }
      if (c + 1 < nmy && !expand_k(c + 1)) break;
      if (!mbar_wait_warp(&bar[SC_DONE + b], (c >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      uint32_t dsr[4 * HG];
      tmem_ld16(tbase + lane_base + kDS0 + b * 32, *(uint32_t(*)[16]) & dsr[0]);
      if (HG > 4) tmem_ld16(tbase + lane_base + kDS0 + b * 32 + 16, *(uint32_t(*)[16]) & dsr[HG > 4 ? 16 : 0]);
      tmem_ld_wait();
      float lg[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        lg[h] = -INFINITY;
        if (h < Hg && live) {
          const long long dot = (long long)(int)dsr[4 * h] + ((long long)(int)dsr[4 * h + 1] << 8) +
                                ((long long)(int)dsr[4 * h + 2] << 16) + ((long long)(int)dsr[4 * h + 3] << 24);
          const float score = nk * fmaf(-2.0f * hcf[2 * h], (float)dot, hcf[2 * h + 1]);
          lg[h] = score * p.scale_log2e;
        }
      }
      // chunk max per head, across the 128 tokens; max |v| (and |v| gamma) for the fixed point
      float mx[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        float v = lg[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        mx[h] = v;
      }
      float vmx = nv, gmx = nv * gm;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        vmx = fmaxf(vmx, __shfl_xor_sync(0xffffffffu, vmx, o));
        gmx = fmaxf(gmx, __shfl_xor_sync(0xffffffffu, gmx, o));
      }
      float* rb = red + (c & 1) * 128;
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < HG; ++h) rb[q * 32 + h] = mx[h];
        rb[q * 32 + 8] = vmx;
        rb[q * 32 + 9] = gmx;
      }
      if (!tok_sync()) break;
      float m2new[HG], corr[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float cm = fmaxf(fmaxf(rb[h], rb[32 + h]), fmaxf(rb[64 + h], rb[96 + h]));
        m2new[h] = fmaxf(m2run[h], cm);
        corr[h] = (m2new[h] == -INFINITY) ? 1.0f : exp2f(m2run[h] - m2new[h]);
      }
      const float U = fmaxf(fmaxf(rb[8], rb[40]), fmaxf(rb[72], rb[104]));
      const float U2 = fmaxf(fmaxf(rb[9], rb[41]), fmaxf(rb[73], rb[105]));
      int E1 = 0, E2 = 0;
      frexpf(fmaxf(U, 1e-30f), &E1);
      frexpf(fmaxf(U2, 1e-30f), &E2);
      const float sw = ldexpf(1.0f, 32 - E1), sw2 = ldexpf(1.0f, 32 - E2);   // w * sw < 2^32
      // weights, their fixed-point limbs (one 32-bit word per head = its four limbs) and sums
      uint32_t wv[HG], wz[HG];
      float sp[HG], sw_[HG], sz_[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float pr = (lg[h] == -INFINITY) ? 0.0f : exp2f(lg[h] - m2new[h]);
        const float w = pr * nv, wg = w * gm;
        wv[h] = __float2uint_rn(w * sw);
        wz[h] = __float2uint_rn(wg * sw2);
        sp[h] = pr;
        sw_[h] = w;
        sz_[h] = wg;
      }
      // the B tiles of the value MMA: token rows of 16 bytes per 4 heads
      if (c >= 2 && !mbar_wait_warp(&bar[V_DONE + b], ((c - 2) >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      uint8_t* bw = smem + Lo.off_bw + (b * 2 + 0) * Lo.bw_bytes;
      uint8_t* bz = smem + Lo.off_bw + (b * 2 + 1) * Lo.bw_bytes;
#pragma unroll
      for (int blk = 0; blk < HG / 4; ++blk) {
        *(uint4*)(bw + blk * kChunk * 16 + t * 16) = make_uint4(wv[4 * blk], wv[4 * blk + 1], wv[4 * blk + 2], wv[4 * blk + 3]);
        *(uint4*)(bz + blk * kChunk * 16 + t * 16) = make_uint4(wz[4 * blk], wz[4 * blk + 1], wz[4 * blk + 2], wz[4 * blk + 3]);
      }
      // chunk sums per head
#pragma unroll
      for (int h = 0; h < HG; ++h) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          sp[h] += __shfl_xor_sync(0xffffffffu, sp[h], o);
          sw_[h] += __shfl_xor_sync(0xffffffffu, sw_[h], o);
          sz_[h] += __shfl_xor_sync(0xffffffffu, sz_[h], o);
        }
      }
      float* rs = red + 256 + (c & 1) * 128;
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          rs[q * 32 + h] = sp[h];
          rs[q * 32 + 8 + h] = sw_[h];
          rs[q * 32 + 16 + h] = sz_[h];
        }
      }
      fence_proxy_async_smem();
      if (!tok_sync()) break;
      // chunk scalars for the accumulators (4-deep ring)
      float* sc = scal + (c & 3) * 64;
      if (q == 0 && lane < HG) {
        const int h = lane;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          a0 += rs[w4 * 32 + h];
          a1 += rs[w4 * 32 + 8 + h];
          a2 += rs[w4 * 32 + 16 + h];
        }
        float ch = 1.0f, mh = 0.0f;
#pragma unroll
        for (int hh = 0; hh < HG; ++hh)
          if (hh == h) {
            ch = corr[hh];
            mh = m2new[hh];
          }
        sc[h] = ch;                 // rescale of the running sums
        sc[8 + h] = a0;             // sum of p
        sc[16 + h] = a1;            // sum of w = p * |v|
        sc[24 + h] = a2;            // sum of w' = p * |v| * gamma
        sc[32 + h] = mh;
        if (h == 0) {
          sc[40] = 1.0f / sw;       // fixed-point scales of the two weight kinds
          sc[41] = 1.0f / sw2;
        }
      }
#pragma unroll
      for (int h = 0; h < HG; ++h) m2run[h] = m2new[h];
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[SCAL_FULL + (c & 3)]);
        mbar_arrive(&bar[BW_FULL + b]);
      }
    }
  } else if (warp < 10) {
    // ------------------------------------ V expanders ----------------------------------------------
    const int t = (warp - 6) * 32 + lane;
    for (int c = 0; c < nmy; ++c) {
      const int st = c % kStages, b = c & 1;
      if (!mbar_wait_warp(&bar[ST_FULL + st], (c / kStages) & 1, p.err, kDevTimeoutLoad, abort_flag)) break;
      if (c >= 2 && !mbar_wait_warp(&bar[V_DONE + b], ((c - 2) >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      const ChunkPos cp = chunk_pos(p, c_begin + c);
      const int tc = (int)min((int64_t)kChunk, T - (int64_t)cp.cis * kChunk);
      const bool live = t < tc;
      const uint8_t* stg = smem + Lo.off_stage + st * Lo.stage_bytes;
      const uint4* vw4 = (const uint4*)((const uint32_t*)(stg + Lo.kc_bytes) + t * 4 * p.bv);
      const uint4* sw4 = (const uint4*)((const uint32_t*)(stg + Lo.kc_bytes + kChunk * 16 * p.bv) + t * 4);
      uint32_t vwr[8];
#pragma unroll
      for (int v4 = 0; v4 < 2; ++v4) {
        uint4 x = make_uint4(0, 0, 0, 0);
        if (v4 < p.bv && live) x = vw4[v4];
        vwr[4 * v4] = x.x;
        vwr[4 * v4 + 1] = x.y;
        vwr[4 * v4 + 2] = x.z;
        vwr[4 * v4 + 3] = x.w;
      }
      uint4 sx = make_uint4(0, 0, 0, 0);
      if (p.vsign && live) sx = *sw4;
      const uint32_t swr[4] = {sx.x, sx.y, sx.z, sx.w};
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t pw[2];
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
          const uint32_t w2 = vwr[2 * g + pl];
          const uint32_t w1 = pl < 1 ? vwr[g] : 0u;
          pw[pl] = p.bv == 2 ? w2 : w1;
        }
#pragma unroll
        for (int P = 0; P < 3; ++P) {
          if (P < p.np) {
            uint32_t w;
            if (p.vsign && P == p.np - 1) {
              w = swr[g];
            } else {
              const int m = p.vmask[P];
              w = ((m & 1) ? pw[0] : 0u) ^ ((m & 2) ? pw[1] : 0u);
            }
            uint8_t* row = smem + Lo.off_av + (b * p.np + P) * Lo.av_bytes;
            const uint4 lo4 = make_uint4(w & 0x01010101u, w & 0x02020202u, w & 0x04040404u, w & 0x08080808u);
            const uint4 hi4 = make_uint4(w & 0x10101010u, w & 0x20202020u, w & 0x40404040u, w & 0x80808080u);
            *(uint4*)(row + sw128_offset(t, g * 32, 128)) = lo4;
            *(uint4*)(row + sw128_offset(t, g * 32 + 16, 128)) = hi4;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[AV_FULL + b]);
        mbar_arrive(&bar[ST_EMPTY + st]);
      }
    }
  } else {
    // ------------------------------------ accumulators (thread = coordinate row) -------------------
    const int q = warp & 3;
    const int m = q * 32 + lane;                 // TMEM lane = M index of the value MMA
    const int g = m >> 5, r = m & 31, s = r >> 2, jj = r & 3;
    const int coord = 32 * g + 8 * jj + s;       // coordinate this row holds
    const float rowscale = ldexpf(1.0f, -s);
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int Hg = p.Hg;
    float acc[3][HG];                            // [value plane][head]
    float Wrun[HG], Zrun[HG], Lrun[HG], Mrun[HG];
    for (int c = 0; c < nmy; ++c) {
      const int b = c & 1;
      const ChunkPos cp = chunk_pos(p, c_begin + c);
      if (seg_first(c)) {
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          acc[0][h] = acc[1][h] = acc[2][h] = 0.0f;
          Wrun[h] = Zrun[h] = Lrun[h] = 0.0f;
          Mrun[h] = -INFINITY;
        }
      }
      if (!mbar_wait_warp(&bar[SCAL_FULL + (c & 3)], (c >> 2) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
      if (!mbar_wait_warp(&bar[V_DONE + b], (c >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      const float* sc = scal + (c & 3) * 64;
      float corr[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        corr[h] = sc[h];
        Lrun[h] = Lrun[h] * corr[h] + sc[8 + h];
        Wrun[h] = Wrun[h] * corr[h] + sc[16 + h];
        Zrun[h] = Zrun[h] * corr[h] + sc[24 + h];
        Mrun[h] = sc[32 + h];
      }
      const float fw = sc[40] * rowscale, fz = sc[41] * rowscale;
#pragma unroll
      for (int P = 0; P < 3; ++P) {
        if (P < p.np) {
          const bool sgn = p.vsign && P == p.np - 1;
          uint32_t dv[4 * HG];
          const uint32_t col = tbase + lane_base + kDV0 + (b * p.np + P) * (4 * HG);
          tmem_ld16(col, *(uint32_t(*)[16]) & dv[0]);
          if (HG > 4) tmem_ld16(col + 16, *(uint32_t(*)[16]) & dv[HG > 4 ? 16 : 0]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < HG; ++h) {
            const unsigned long long y = (unsigned long long)dv[4 * h] + ((unsigned long long)dv[4 * h + 1] << 8) +
                                         ((unsigned long long)dv[4 * h + 2] << 16) +
                                         ((unsigned long long)dv[4 * h + 3] << 24);
            acc[P][h] = fmaf(acc[P][h], corr[h], (float)y * (sgn ? fz : fw));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[DV_EMPTY + b]);
      if (seg_last(c)) {
        // fold the Walsh planes and write this segment's partial state
        const int sg = cp.slice;
        const int seg = (c_begin + c) / p.per_cta - (sg * p.nchunk) / p.per_cta;   // CTA ordinal inside the slice
        float* rec = p.partial + ((size_t)sg * p.maxseg + seg) * Hg * att_rec(d);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          if (h < Hg) {
            float* rh = rec + h * att_rec(d);
            float om = 0.0f;
#pragma unroll
            for (int P = 0; P < 3; ++P)
              if (P < p.mv) om += p.beta_v[P] * (Wrun[h] - 2.0f * acc[P][h]);
            float oz = 0.0f;
#pragma unroll
            for (int P = 0; P < 3; ++P)
              if (p.vsign && P == p.np - 1) oz = 2.0f * acc[P][h] - Zrun[h];
            rh[4 + coord] = om;
            rh[4 + d + coord] = oz;
            if (m == 0) {
              rh[0] = Mrun[h];
              rh[1] = Lrun[h];
              rh[2] = 1.0f;                       // marks a written record
              rh[3] = 0.0f;
            }
          }
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

// ------------------------------------------------------------------------------------------------
// combine: merge the partial states of a slice, apply Pi^T and alpha S^T once per query head
// ------------------------------------------------------------------------------------------------
__global__ void attend_combine_kernel(const __grid_constant__ AttParams p) {
  const int bh = blockIdx.x;                 // b * Hq + hq
  const int b = bh / p.Hq, hq = bh % p.Hq;
  const int hk = hq / p.Hg, h = hq % p.Hg;
  const int slice = b * p.Hkv + hk;
  const int d = p.d, i = threadIdx.x;
  __shared__ float orot[128], osgn[128];
  __shared__ float mmax, linv;
  // CTAs that touched this slice
  const int first = (slice * p.nchunk) / p.per_cta;
  const int last = (slice * p.nchunk + p.nchunk - 1) / p.per_cta;
  const int nseg = last - first + 1;
  const float* base = p.partial + (size_t)slice * p.maxseg * p.Hg * att_rec(d) + (size_t)h * att_rec(d);
  const size_t stride = (size_t)p.Hg * att_rec(d);
  if (i == 0) {
    float M = -INFINITY;
    for (int sgi = 0; sgi < nseg; ++sgi) M = fmaxf(M, base[sgi * stride]);
    float L = 0.0f;
    for (int sgi = 0; sgi < nseg; ++sgi) {
      const float ms = base[sgi * stride];
      if (ms > -INFINITY) L += base[sgi * stride + 1] * exp2f(ms - M);
    }
    mmax = M;
    linv = L > 0.0f ? 1.0f / L : 0.0f;
  }
  __syncthreads();
  if (i < d) {
    float a = 0.0f, z = 0.0f;
    for (int sgi = 0; sgi < nseg; ++sgi) {
      const float ms = base[sgi * stride];
      if (ms == -INFINITY) continue;
      const float f = exp2f(ms - mmax);
      a = fmaf(base[sgi * stride + 4 + i], f, a);
      z = fmaf(base[sgi * stride + 4 + d + i], f, z);
    }
    orot[i] = a * linv;
    osgn[i] = z * linv;
  }
  __syncthreads();
  if (i < d) {
    float acc = 0.0f;
    for (int j = 0; j < d; ++j) acc = fmaf(p.Pi[(size_t)j * d + i], orot[j], acc);
    if (p.vsign) {
      float a2 = 0.0f;
      for (int j = 0; j < d; ++j) a2 = fmaf(p.S[(size_t)j * d + i], osgn[j], a2);
      acc = fmaf(p.alpha, a2, acc);
    }
    p.out[(size_t)bh * d + i] = acc;
  }
}

// Walsh coefficients of an exactly symmetric codebook over the odd subsets of its bit planes.
int walsh_planes(const tq_codebook* cb, int* mask, float* beta) {
  const int L = cb->levels, bits = cb->bits;
  int n = 0;
  for (int m = 1; m < (1 << bits); ++m) {
    if (!(__builtin_popcount(m) & 1)) continue;
    double acc = 0.0;
    for (int idx = 0; idx < L; ++idx) {
      int par = __builtin_popcount(idx & m) & 1;            // XOR of the planes in the subset
      acc += (double)cb->c[idx] * (par ? -1.0 : 1.0);       // prod (1 - 2 bit) = 1 - 2 parity
    }
    mask[n] = m;
    beta[n] = (float)(acc / L);
    ++n;
  }
  return n;
}

struct AttPlan {
  AttParams p;
  size_t bq_bytes, hc_bytes, part_bytes, total;
};

bool att_plan(int B, int Hq, int Hkv, int64_t T, int d, int nsm, AttPlan& pl) {
  AttParams& p = pl.p;
  p = AttParams{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Hg = Hq / Hkv;
  p.d = d;
  p.G = d / 32;
  p.T = T;
  p.slices = B * Hkv;
  p.nchunk = (int)((T + kChunk - 1) / kChunk);
  const long long totalc = (long long)p.slices * p.nchunk;
  const int ncta = (int)std::min<long long>(nsm, totalc);
  p.per_cta = (int)((totalc + ncta - 1) / ncta);
  p.maxseg = (p.nchunk + p.per_cta - 1) / p.per_cta + 1;
  p.nq = p.Hg <= 4 ? 16 : 32;      // the kernel is built for 4 or 8 heads per KV head
  p.nvc = p.nq;
  pl.bq_bytes = (size_t)p.slices * p.nq * 4 * d;       // mk <= 4
  pl.hc_bytes = (size_t)p.slices * 16 * sizeof(float);
  pl.part_bytes = (size_t)p.slices * p.maxseg * p.Hg * att_rec(d) * sizeof(float);
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  pl.total = al(pl.bq_bytes) + al(pl.hc_bytes) + al(pl.part_bytes);
  return true;
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" TQ_API size_t tq_attend_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t T, int32_t d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || Hq % Hkv) return 0;
  // the split of the chunks over CTAs depends on the SM count of the current device
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      nsm <= 0) {
    cudaGetLastError();
    nsm = 148;
  }
  AttPlan pl;
  att_plan(B, Hq, Hkv, T, d, nsm, pl);
  return pl.total;
}

extern "C" TQ_API tq_status tq_attend_decode(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                             int32_t Hkv, int64_t T, int32_t d, const void* q, int32_t q_dtype,
                                             const void* rot, const uint32_t* k_codes, const uint16_t* k_norms,
                                             const uint32_t* v_codes, const uint32_t* v_signs, const uint16_t* v_norms,
                                             const uint16_t* v_gammas, float scale, float* out, void* ws,
                                             size_t ws_bytes, void* stream) {
  clear_error();
  const char* f = "tq_attend_decode";
  if (!cb_k || !cb_v || !q || !rot || !k_codes || !k_norms || !v_codes || !v_norms || !out || !ws)
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": NULL pointer");
  if ((v_signs == nullptr) != (v_gammas == nullptr))
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": v_signs and v_gammas must both be NULL or both be set");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || Hq % Hkv)
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": bad B / Hq / Hkv / T");
  if (d != 128) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": this build supports d = 128");
  if (Hq / Hkv > 8) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": at most 8 query heads per KV head");
  if (T > ((int64_t)1 << 31)) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": T too large");
  if (cb_k->d != d || cb_v->d != d) return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": codebook d mismatch");
  if (cb_k->bits < 1 || cb_k->bits > 3)
    return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": key codebooks of 1..3 bits are supported");
  const bool vsign = v_signs != nullptr;
  if (cb_v->bits < 1 || cb_v->bits > 2)   // value planes (Walsh planes + sign) must fit three MMA operand slots
    return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": value codebooks of 1..2 bits are supported");
  for (const tq_codebook* cb : {cb_k, cb_v}) {
    const int L = cb->levels;
    if (L != (1 << cb->bits)) return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": bad codebook");
    for (int k = 0; k < L; ++k)
      if (cb->c[L - 1 - k] != -cb->c[k]) return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": codebook not symmetric");
  }
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": q dtype");
  if (!aligned16(k_codes) || !aligned16(v_codes) || (vsign && !aligned16(v_signs)) || !aligned16(ws) ||
      !aligned16(rot) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": pointers must be 16-byte aligned");
  AttPlan pl;
  att_plan(B, Hq, Hkv, T, d, sm_count(), pl);
  if (ws_bytes < pl.total || ws_bytes < tq_attend_workspace_bytes(B, Hq, Hkv, T, d))
    return fail(TQ_ERR_WORKSPACE, std::string(f) + ": workspace too small");
  AttParams& p = pl.p;
  p.bk = cb_k->bits;
  p.mk = walsh_planes(cb_k, p.kmask, p.beta_k);
  p.bv = cb_v->bits;
  p.mv = walsh_planes(cb_v, p.vmask, p.beta_v);
  p.vsign = vsign ? 1 : 0;
  p.np = p.mv + p.vsign;
  if (p.np > 3) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": too many value planes");
  p.scale_log2e = scale * kLog2e;
  p.alpha = (float)(std::sqrt(M_PI / 2.0) / d);
  p.q = q;
  p.q_bf16 = q_dtype == TQ_BF16;
  RotLayout RL = rot_layout(d);
  p.Pi = (const float*)((const char*)rot + RL.pi32);
  p.S = (const float*)((const char*)rot + RL.s32);
  p.k_codes = k_codes;
  p.k_norms = k_norms;
  p.v_codes = v_codes;
  p.v_signs = v_signs;
  p.v_norms = v_norms;
  p.v_gammas = v_gammas;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* w = (uint8_t*)ws;
  p.bq_img = w;
  p.head_c = (float*)(w + al(pl.bq_bytes));
  p.partial = (float*)(w + al(pl.bq_bytes) + al(pl.hc_bytes));
  p.out = out;
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, std::string(f) + ": no device error word");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  attend_prep_kernel<<<p.slices, 128, 0, st>>>(p);
  const AttLayout Lo = att_layout(p);
  auto kern = p.Hg <= 4 ? attend_main_kernel<4> : attend_main_kernel<8>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "tq_attend_decode: shared memory attribute");
  const long long totalc = (long long)p.slices * p.nchunk;
  const int grid = (int)((totalc + p.per_cta - 1) / p.per_cta);
  kern<<<grid, kAttThreads, Lo.total, st>>>(p);
  attend_combine_kernel<<<B * Hq, 128, 0, st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tq_attend_decode: launch");
  return TQ_OK;
}
