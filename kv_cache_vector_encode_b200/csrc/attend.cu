// Decode attention over a TurboQuant-packed KV cache (tq_attend_decode).
//
// Method (aiboss88 page: attention evaluated on the quantised cache, unbiased inner-product
// estimates; ai-navigate-news page: keys by Algorithm 1, values by Algorithm 2):
//   out[b][h] = sum_t softmax_t(scale <q, k_hat_t>) v_hat_t,   k_hat_t = n_t Pi^T c_K[idx_t],
//   v_hat_t = m_t (Pi^T c_V[jdx_t] + alpha gamma_t S^T (2 z_t - 1)).
// Keys may also be Algorithm 2: k_hat_t = n_t (Pi^T c_K[idx_t] + alpha g_t S^T (2 y_t - 1)), whose
// extra score term alpha g_t <S q, 2 y_t - 1> is one more 0 / 2^s plane (the key sign bits) against
// the fixed-point digits of q'' = S q, accumulated into score columns of its own.
// Evaluated from the codes, never materialising k_hat or v_hat:
//   * the query is rotated once, q' = Pi q (and projected, q'' = S q, for Algorithm 2 keys) (prep
//     kernel);
//   * the codebook is an odd function of the index bits (exact symmetry), so c[idx] =
//     sum_S beta_S prod_{p in S} (1 - 2 bit_p) over the odd subsets S of the bit planes
//     (Walsh expansion). With b_S = XOR of the planes in S,
//       <q', c[idx]> = sum_S beta_S (Q - 2 <q', b_S>),   Q = sum_i q'_i,
//     and <q', b_S> is an exact integer tensor-core product: A = the bits b_S (0/1 bytes, scaled
//     by 2^s, see below), B = beta_S q' in 32-bit fixed point as four signed 8-bit limbs;
//   * values are accumulated in the rotated / sign domain. For each value plane P (the Walsh
//     planes of the value codes, then the sign plane) the value MMA gives Y_P[i] = sum_t w_t b_P,t,i
//     with the softmax weights w_t (times the value norm, times gamma for the sign plane) in 32-bit
//     unsigned fixed point (24 bits) as 8-bit limbs. Over a run of chunks with unchanged maxima and
//     scales, the value MMAs accumulate Y_P in TMEM, and the value MMA warp adds up the run's weights
//     W = sum_t w_t (and W' of the sign plane) exactly from the same weight tiles; the folds
//       O_P = sum_t w_t (1 - 2 b_P,t) = W - 2 Y_P,   O_z = sum_t w'_t (2 z_t - 1) = 2 Y_z - W'
//     are formed once per run before the running (rescaled) accumulation;
//   * once per query head: out = (Pi^T sum_P beta_P O_P + alpha S^T O_z) / sum_t p_t.
//
// Bit expansion: a 32-bit plane word w covers 32 coordinates; register s (s = 0..7) of
// (w & (0x01010101 << s)) holds coordinates s, 8+s, 16+s, 24+s as bytes 0 or 2^s. The tensor-core
// index order inside each 32-coordinate group is therefore k = 4 s + j for coordinate 8 j + s,
// and the 2^s factor is divided out of the query limbs (scores) or of the output rows (values).
//
// Online softmax: a running maximum per head and running maxima of the value weights (which fix
// the fixed-point scales). A chunk needs a group's four softmax warps to exchange maxima only when some
// token exceeds a running maximum; one barrier with an OR-reduction decides that, so after the
// first chunks of a segment most chunks take no exchange at all.
//
// Kernels: prep (q' limbs, per-head constants), main (persistent; one CTA per SM walks a
// contiguous range of 128-token chunks, possibly spanning several (batch, KV head) slices), combine
// (merges the per-CTA partial states of a slice and applies Pi^T, S^T).
// Main-kernel roles (19 warps): 0 bulk-copies packed chunks; 1 owns TMEM and issues the key MMAs;
// then the softmax warps (thread = token; one group of four warps per four query heads: 2-5, or
// 2-9 with eight heads); then four warps that expand the key planes into TMEM (thread = token), and
// with eight heads also the value planes into shared memory; four warps that accumulate the value
// products (thread = coordinate); one that issues the value MMAs; and with four heads, four more
// that expand the value planes, so that key and value expansion run side by side.
// All mbarrier waits are bounded (sm100.cuh); the softmax warps' named barriers are reached the
// same number of times by the four warps of a group (their loop never exits early).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <vector>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

// warps of the main kernel: 23 when the value planes have their own expander warps (at most four
// query heads per KV head; 80 registers a thread), else 19 (96 registers)
__host__ __device__ constexpr bool att_split_v(int hg) { return hg <= 4; }
// softmax groups of four warps: one per four query heads
__host__ __device__ constexpr int att_groups(int hg) { return hg / 4; }
// producer, key MMA, softmax groups, key (and value) expanders, accumulators, value MMA, and with at
// most four query heads separate value expanders: 19 warps either way
__host__ __device__ constexpr int att_warps(int hg) { return 2 + 4 * att_groups(hg) + 8 + 1 + (att_split_v(hg) ? 4 : 0); }
constexpr int kChunk = 128;                 // tokens per chunk
constexpr int kMaxStages = 8;               // packed-chunk ring (depth chosen from shared memory)
constexpr int kMaxSmem = 232448;            // 227 KB of dynamic shared memory per block
constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------------------------------------
// Parameters shared by the three kernels
// ------------------------------------------------------------------------------------------------
struct AttParams {
  int B, Hq, Hkv, d, G;
  // Virtual heads: a pass attends Hg = nqry x Hgr (query token, query head) pairs per slice; query
  // token j of the pass and head h are virtual head j * Hgr + h. Decode has nqry = 1 (Hg = Hgr).
  int Hg, Hgr, nqry;
  int64_t q_bs, q_js;            // element strides of q and out: batch, query token (head stride d)
  int64_t tlim0;                 // query token j attends the tokens t < tlim0 + j
  // A launch may hold several passes: work slice s is pass s / cslices over cache slice s % cslices
  // (b * Hkv + hk); pass ps serves query tokens ps * nqry .. ps * nqry + nqry - 1 of nqtot.
  int cslices, nqtot;
  int64_t T;                     // tokens attended per slice
  int64_t tstride;               // token slots per slice in the cache arrays (>= T)
  int slices, nchunk, per_cta, maxseg;   // work slices (passes x cache slices), chunks per slice
  int nst;                       // depth of the packed-chunk ring
  int norm_bulk;                 // 1: the norm arrays are bulk-copied into the stage with the codes
                                 // (slot stride a multiple of 8 tokens, 16-byte aligned arrays)
  int bk, mk, ksign;             // key codebook bits, key Walsh planes, key sign plane (Algorithm 2 keys)?
  int bv, mv, vsign, np;         // value codebook bits, value Walsh planes, sign plane?, planes
  int nq;                        // MMA N of the scores / of one value weight kind (16 or 32)
  float beta_k[4], beta_v[4];
  float scale_log2e, alpha;
  const void* q;
  int q_bf16;
  const float* Pi;
  const float* S;
  const uint32_t* k_codes;
  const uint16_t* k_norms;
  const uint32_t* k_signs;       // Algorithm 2 keys only (else NULL)
  const uint16_t* k_gammas;
  const uint32_t* v_codes;
  const uint32_t* v_signs;
  const uint16_t* v_norms;
  const uint16_t* v_gammas;
  // append (tq_attend_append): the prep kernel encodes each slice's new key (Algorithm 1) and value
  // (Algorithm 2) into slot t_new of the cache before the main kernel reads it; NULL otherwise
  const void* k_new;
  const void* v_new;             // [slices][d], x_bf16 ? bf16 : fp32
  int x_bf16;
  int64_t t_new;
  uint32_t* kw_codes;
  uint16_t* kw_norms;
  uint32_t* vw_codes;
  uint32_t* vw_signs;
  uint16_t* vw_norms;
  uint16_t* vw_gammas;
  float ck[8], tk[8], cv[8], tv[8];   // fp32 centroids / boundaries of the key and value codebooks
  uint8_t* bq_img;               // [slices][nq rows x (mk + ksign) d bytes] K-major SW128 image
  float* head_c;                 // [slices][8][4]: 2^-F, Q_h * sum beta, 2^-F'', Q''_h
  float* partial;                // [slices][maxseg][Hg][att_rec(d)]
  float* out;
  uint32_t* err;
};

// partial record of one (segment, head): [0] running max (log2 domain), [1] sum of p, [2] 1 when
// written, [3] unused, then the folded value planes O_P[d] for P = 0..2
__host__ __device__ inline int att_rec(int d) { return 4 + 3 * d; }

// ------------------------------------------------------------------------------------------------
// append: encode one new vector of a slice into its cache slot, in fp64 on the SIMT cores (thread =
// coordinate, 128 threads). The steps are Algorithm 1 / 2 as the encoders compute them (ai-navigate-
// news page, "how it works (technical)"): n = |x| (fp16 record), u = x / n (zero and non-finite rows:
// u = 0), y = Pi u, idx_j = #{k : t_k < y_j}, bit planes by ballot; Algorithm 2 adds
// r = u - Pi^T c[idx], gamma = |r| and the sign bits of S r.
// ------------------------------------------------------------------------------------------------
__device__ double prep_block_sum(double v, double* red4) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red4[warp] = v;
  __syncthreads();
  return (red4[0] + red4[1]) + (red4[2] + red4[3]);
}

__device__ void append_encode(const AttParams& p, int slice, const void* xsrc, bool alg2, int bits, const float* c,
                              const float* t, uint32_t* codes, uint16_t* norms, uint32_t* signs, uint16_t* gammas,
                              double* sh, double* red4) {
  const int d = p.d, i = threadIdx.x, g = i >> 5, lane = i & 31;
  const int L = 1 << bits;
  const size_t xo = (size_t)slice * d + i;
  const double xi = p.x_bf16 ? (double)__uint_as_float((uint32_t)((const uint16_t*)xsrc)[xo] << 16)
                             : (double)((const float*)xsrc)[xo];
  const double n = sqrt(prep_block_sum(xi * xi, red4));
  const bool ok = isfinite(n) && n > 0.0;
  double* u = sh;                                     // [128]
  double* cs = sh + 128;                              // [128]
  u[i] = ok ? xi / n : 0.0;
  __syncthreads();
  double y = 0.0;                                     // y_i = sum_j Pi[i][j] u_j
  for (int j = 0; j < d; ++j) y = fma((double)__ldg(p.Pi + (size_t)i * d + j), u[j], y);
  int idx = 0;
  for (int k = 0; k < L - 1; ++k) idx += (double)t[k] < y ? 1 : 0;
  const int64_t rec = (int64_t)slice * p.tstride + p.t_new;
  for (int pl = 0; pl < bits; ++pl) {
    const uint32_t w = __ballot_sync(0xffffffffu, (idx >> pl) & 1);
    if (lane == 0) codes[(rec * p.G + g) * bits + pl] = w;
  }
  if (i == 0) norms[rec] = __half_as_ushort(__double2half(n));
  if (!alg2) return;
  cs[i] = (double)c[idx];
  __syncthreads();
  double a = 0.0;                                     // (Pi^T c)_i = sum_j Pi[j][i] c_j
  for (int j = 0; j < d; ++j) a = fma((double)__ldg(p.Pi + (size_t)j * d + i), cs[j], a);
  const double r = ok ? u[i] - a : 0.0;
  const double gam = sqrt(prep_block_sum(r * r, red4));
  cs[i] = r;                                          // (the sums above synchronised the block)
  __syncthreads();
  double sv = 0.0;                                    // (S r)_i
  for (int j = 0; j < d; ++j) sv = fma((double)__ldg(p.S + (size_t)i * d + j), cs[j], sv);
  const uint32_t w = __ballot_sync(0xffffffffu, sv >= 0.0);
  if (lane == 0) signs[rec * p.G + g] = w;
  if (i == 0) gammas[rec] = __half_as_ushort(__double2half(gam));
  __syncthreads();
}

// ------------------------------------------------------------------------------------------------
// prep: q' = Pi q per query head, fixed-point limbs of beta_S q' (scaled by 2^-s), constants
// ------------------------------------------------------------------------------------------------
constexpr int kPrepRow = 129;                   // staged matrix row (floats): row reads hit distinct banks
size_t prep_smem_bytes(int ksign) { return (size_t)(ksign ? 2 : 1) * 128 * kPrepRow * sizeof(float); }

__global__ void attend_prep_kernel(const __grid_constant__ AttParams p) {
  extern __shared__ float prep_mat[];           // Pi, then S (Algorithm 2 keys): [128][kPrepRow]
  grid_dep_launch();                            // the main kernel may be scheduled (it waits for this grid)
  const int slice = blockIdx.x;                  // work slice: pass * cslices + b * Hkv + hk
  const int cs = slice % p.cslices, ps = slice / p.cslices;
  const int b = cs / p.Hkv, hk = cs % p.Hkv;
  const int d = p.d, i = threadIdx.x;            // coordinate (128 threads)
  const int warp = i >> 5, lane = i & 31;
  __shared__ __align__(16) float sq[8][128];
  __shared__ double red[4][8][4];
  if (p.kw_codes) {
    // append: this slice's new key and value go into slot t_new before anything reads the cache
    __shared__ double esh[256];
    __shared__ double ered[4];
    append_encode(p, slice, p.k_new, false, p.bk, p.ck, p.tk, p.kw_codes, p.kw_norms, nullptr, nullptr, esh, ered);
    append_encode(p, slice, p.v_new, true, p.bv, p.cv, p.tv, p.vw_codes, p.vw_norms, p.vw_signs, p.vw_gammas, esh,
                  ered);
  }
  const int kbytes = (p.mk + p.ksign) * d;
  uint8_t* img = p.bq_img + (size_t)slice * p.nq * kbytes;
  for (int o = i; o < p.nq * kbytes / 16; o += blockDim.x) ((uint4*)img)[o] = make_uint4(0, 0, 0, 0);
  for (int h = 0; h < p.Hg; ++h) {
    const int j = ps * p.nqry + h / p.Hgr;       // query token of virtual head h (none past nqtot)
    const size_t qoff = (size_t)b * p.q_bs + (size_t)j * p.q_js + (size_t)(hk * p.Hgr + h % p.Hgr) * d;
    sq[h][i] = j >= p.nqtot ? 0.0f
                            : (p.q_bf16 ? __uint_as_float((uint32_t)((const uint16_t*)p.q)[qoff + i] << 16)
                                        : ((const float*)p.q)[qoff + i]);
  }
  // Pi (and S) into shared memory: coalesced 16-byte loads, all in flight at once, stored into
  // padded rows
  for (int mtx = 0; mtx < (p.ksign ? 2 : 1); ++mtx) {
    const float4* src = (const float4*)(mtx ? p.S : p.Pi);
    float* dst = prep_mat + mtx * 128 * kPrepRow;
#pragma unroll 8
    for (int o = i; o < 128 * 32; o += 128) {
      const float4 v = __ldg(src + o);
      float* q = dst + (o >> 5) * kPrepRow + (o & 31) * 4;
      q[0] = v.x;
      q[1] = v.y;
      q[2] = v.z;
      q[3] = v.w;
    }
  }
  __syncthreads();
  // q'_h[i] = sum_j Pi[i][j] q_h[j] for every head: one thread per output coordinate, its row of Pi
  // from shared memory, fp64 accumulation (one independent chain per head)
  // (q''_h = S q_h the same way, for Algorithm 2 keys)
  double acc[8], acc2[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) acc[h] = acc2[h] = 0.0;
  const float* row = prep_mat + i * kPrepRow;
  const float* srow = prep_mat + 128 * kPrepRow + i * kPrepRow;
#pragma unroll 4
  for (int j = 0; j < 128; ++j) {
    const double pv = (double)row[j];
    const double sv = p.ksign ? (double)srow[j] : 0.0;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < p.Hg) {
        const double qv = (double)sq[h][j];
        acc[h] = fma(pv, qv, acc[h]);
        if (p.ksign) acc2[h] = fma(sv, qv, acc2[h]);
      }
    }
  }
  double bmax = 0.0, sb = 0.0;
  for (int S = 0; S < p.mk; ++S) {
    bmax = fmax(bmax, fabs((double)p.beta_k[S]));
    sb += (double)p.beta_k[S];
  }
  // per head: Q_h = sum_i q'_i and max_i |q'_i| bmax, warp shuffles then one exchange
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < p.Hg) {
      double sm = acc[h], mx = fabs(acc[h]) * bmax, sm2 = acc2[h], mx2 = fabs(acc2[h]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sm += __shfl_xor_sync(0xffffffffu, sm, o);
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        sm2 += __shfl_xor_sync(0xffffffffu, sm2, o);
        mx2 = fmax(mx2, __shfl_xor_sync(0xffffffffu, mx2, o));
      }
      if (lane == 0) {
        red[warp][h][0] = sm;
        red[warp][h][1] = mx;
        red[warp][h][2] = sm2;
        red[warp][h][3] = mx2;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h >= p.Hg) break;
    const double qi = acc[h];
    const double Qh = (red[0][h][0] + red[1][h][0]) + (red[2][h][0] + red[3][h][0]);
    const double vmax = fmax(fmax(red[0][h][1], red[1][h][1]), fmax(red[2][h][1], red[3][h][1]));
    int F = 0;
    if (vmax > 0.0) {
      int E;
      frexp(vmax, &E);              // vmax < 2^E
      F = 30 - E;                   // vmax * 2^F < 2^30
    }
    // q'' of Algorithm 2 keys: fixed point 2^F2 with max |q''| 2^F2 < 2^30
    const double Q2 = (red[0][h][2] + red[1][h][2]) + (red[2][h][2] + red[3][h][2]);
    const double vmax2 = fmax(fmax(red[0][h][3], red[1][h][3]), fmax(red[2][h][3], red[3][h][3]));
    int F2 = 0;
    if (vmax2 > 0.0) {
      int E;
      frexp(vmax2, &E);
      F2 = 30 - E;
    }
    if (i == 0) {
      p.head_c[(slice * 8 + h) * 4 + 0] = (float)ldexp(1.0, -F);
      p.head_c[(slice * 8 + h) * 4 + 1] = (float)(Qh * sb);
      p.head_c[(slice * 8 + h) * 4 + 2] = (float)ldexp(1.0, -F2);
      p.head_c[(slice * 8 + h) * 4 + 3] = (float)Q2;
    }
    const int g = i >> 5, rr = i & 31, jj = rr >> 3, s = rr & 7;   // coordinate 32g + 8jj + s
    const int kin = 32 * g + 4 * s + jj;                          // its k index inside a plane
    for (int S = 0; S < p.mk + p.ksign; ++S) {
      // the Walsh planes carry beta_S q'; the key sign plane (last) carries q''
      long long v = S < p.mk ? llrint(ldexp((double)p.beta_k[S] * qi, F - s)) : llrint(ldexp(acc2[h], F2 - s));
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
// A run is a stretch of consecutive chunks of one slice over which no running maximum and no
// fixed-point scale of the softmax changes: the value MMAs accumulate its chunks in one TMEM buffer
// (exact int32 limb sums) and the accumulator warps fold it once. Runs stop at 256 chunks, which
// keeps every limb sum below 2^30. Run record (kRunRec bytes): [0, 32) running maxima of the 8
// heads, [32] 1/sw, [36] 1/sw', [40] flags (1 = last run of its segment, 2 = last run of the CTA),
// [44] segment ordinal, [48] slice, [64, 192) exact run sums (uint64) of the weight kinds w and
// w gamma for the 8 heads, [192, 224) the segment's sums of p for the 8 heads (last run of a
// segment only).
constexpr int kRunRec = 256;
constexpr int kMaxRun = 256;

struct AttLayout {
  uint32_t kc_bytes, vc_bytes, sg_off, ks_off, nrm_off, stage_bytes;
  uint32_t off_stage, av_bytes, off_av, bw_kind, bw_buf, off_bw, bq_bytes, off_bq, off_sc, off_red, off_sum,
      off_run, off_bar, total;
};

__host__ __device__ inline uint32_t aru(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline AttLayout att_layout(const AttParams& p, int nst) {
  AttLayout L{};
  L.kc_bytes = kChunk * p.G * p.bk * 4;
  L.sg_off = L.kc_bytes + kChunk * p.G * p.bv * 4;     // sign words of the chunk
  L.vc_bytes = kChunk * p.G * (p.bv + (p.vsign ? 1 : 0)) * 4;
  L.ks_off = L.kc_bytes + L.vc_bytes;                 // key sign words (Algorithm 2 keys)
  // fp16 key norms, value norms, value gammas, key gammas of the chunk: [4][128]
  L.nrm_off = aru(L.ks_off + (p.ksign ? kChunk * p.G * 4 : 0), 16);
  L.stage_bytes = aru(L.nrm_off + (p.norm_bulk ? 4 * kChunk * 2 : 0), 1024);
  uint32_t off = 0;
  L.off_stage = off; off += nst * L.stage_bytes;
  L.av_bytes = kChunk * 128;                       // one plane: 128 tokens x 128 coordinates
  L.off_av = off; off += 3 * p.np * L.av_bytes;     // three chunks of value planes
  L.bw_kind = (p.nq / 16) * kChunk * 16;           // one weight kind: nq/16 blocks of 128 x 16 bytes
  L.bw_buf = 2 * L.bw_kind;                        // kinds: w, w * gamma
  L.off_bw = off; off += 2 * L.bw_buf;
  L.bq_bytes = aru(p.nq * (p.mk + p.ksign) * p.d, 1024);
  L.off_bq = off; off += 2 * L.bq_bytes;
  L.off_sc = off; off += 4 * 64 * 4;               // chunk scalars, 4-deep ring of 64 floats
  L.off_red = off; off += 2 * 4 * 16 * 4;          // max exchange of the softmax warps: [group][warp][16]
  L.off_sum = off; off += 4 * 4 * 8 * 4;           // segment sums of p: [4 slots][warp][head]
  L.off_run = aru(off, 16); off = L.off_run + 2 * kRunRec;   // records of the two runs in flight
  L.off_bar = aru(off, 8); off = L.off_bar + 64 * 8;
  L.total = off + 1024;
  return L;
}


enum ABars {
  ST_FULL = 0,                         // [kMaxStages]
  ST_EMPTY = ST_FULL + kMaxStages,     // [kMaxStages] (key and value expander warps, 4 or 8, and the
                                       //  8 softmax warps, which read the stage's norms)
  BQ_FULL = ST_EMPTY + kMaxStages,     // [2]
  BQ_EMPTY = BQ_FULL + 2,              // [2]
  AK_FULL = BQ_EMPTY + 2,              // [2]  key expanders -> key MMA warp: key planes in TMEM (4 warps)
  SC_DONE = AK_FULL + 2,               // [2]  scores MMA complete (commit)
  BW_FULL = SC_DONE + 2,               // [2]  softmax -> MMA warps (8 warps)
  AV_FULL = BW_FULL + 2,               // [3]  value expanders -> value MMA warp: value planes (4 warps)
  V_DONE = AV_FULL + 3,                // [6]  value MMA of chunk c complete (commit), slot c % 6
  RUN_DONE = V_DONE + 6,               // [2]  value MMA warp -> accumulators: a run's MMAs complete (commit)
                                       //      and its record written (arrive): 2 arrivals
  RUN_FREE = RUN_DONE + 2,             // [2]  accumulators -> value MMA warp: run buffer drained (4 warps)
  SC_FREE = RUN_FREE + 2,              // [2]  softmax -> key MMA warp: scores buffer read (8 warps)
  ANBARS = SC_FREE + 2
};

// TMEM columns: A_K [2][32 (mk + ksign)] at 0, scores [2][nq (1 + ksign)] after them, value
// accumulators [2][np][nq] after those (at most 512 columns: mk + ksign <= 4 and with a key sign
// plane mk <= 2).

// Walks this CTA's chunks in order (slice, chunk inside the slice, segment ordinal) without
// integer division.
struct ChunkIter {
  int slice, cis, seg, nchunk, cs, ncs;   // work slice, chunk in it, segment ordinal; cache slice
  __device__ __forceinline__ void init(const AttParams& p, int gchunk) {
    nchunk = p.nchunk;
    slice = gchunk / nchunk;
    cis = gchunk - slice * nchunk;
    seg = 0;
    ncs = p.cslices;
    cs = slice % ncs;
  }
  __device__ __forceinline__ void next() {
    if (++cis == nchunk) {
      cis = 0;
      ++slice;
      ++seg;
      if (++cs == ncs) cs = 0;
    }
  }
};

// Position in a ring of n slots walked one step per chunk: slot and the parity of the pass over the
// ring (the mbarrier phase), kept incrementally instead of by division.
struct RingPos {
  int slot, n;
  uint32_t par;
  __device__ __forceinline__ void next() {
    if (++slot == n) {
      slot = 0;
      par ^= 1u;
    }
  }
};

// odd subsets of `bits` bit planes in increasing order (the Walsh planes of a symmetric codebook)
__host__ __device__ constexpr int walsh_count(int bits) { return bits == 1 ? 1 : (bits == 2 ? 2 : 4); }
__host__ __device__ constexpr int walsh_mask(int bits, int S) {
  return bits == 3 ? (S == 0 ? 1 : (S == 1 ? 2 : (S == 2 ? 4 : 7))) : (S == 0 ? 1 : 2);
}

// l0 + 2^8 l1 + 2^16 l2 + 2^24 l3 for signed limb sums |l| < 2^21: the pairs are exact in 32 bits
// (|l0 + 2^8 l1| < 2^30), then two conversions and one FMA.
__device__ __forceinline__ float limbs_to_float(uint32_t l0, uint32_t l1, uint32_t l2, uint32_t l3) {
  const int lo = (int)l0 + (int)(l1 << 8);
  const int hi = (int)l2 + (int)(l3 << 8);
  return fmaf((float)hi, 65536.0f, (float)lo);
}

// Round-to-nearest of 0 <= v <= 2^23 to an integer with one FMA (v = a * b).
__device__ __forceinline__ uint32_t fixed24(float a, float b) {
  return __float_as_uint(fmaf(a, b, 8388608.0f)) - 0x4B000000u;
}

// 2^x with the hardware approximation (ex2.approx.ftz; |relative error| about 2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.add.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}
// exact warp sum of values below 2^43: the low 16 bits and the rest are reduced separately
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
  const uint32_t lo = warp_sum_u32((uint32_t)v & 0xFFFFu), hi = warp_sum_u32((uint32_t)(v >> 16));
  return ((unsigned long long)hi << 16) + lo;
}

// Value planes of one token (thread = token t of the chunk): plane words (and sign words) ->
// bytes 0 / 2^s, one 128-byte token row per plane (128-byte swizzle, slots voff).
template <int BV, int VS, int NP>
__device__ __forceinline__ void expand_v_rows(const AttParams& p, const AttLayout& Lo, const uint8_t* stg, uint8_t* avb,
                                              int t, const uint32_t (&voff)[8]) {
  uint32_t vw[4 * BV];
#pragma unroll
  for (int v4 = 0; v4 < BV; ++v4) {
    const uint4 x = *(const uint4*)(stg + Lo.kc_bytes + t * 16 * BV + v4 * 16);
    vw[4 * v4] = x.x;
    vw[4 * v4 + 1] = x.y;
    vw[4 * v4 + 2] = x.z;
    vw[4 * v4 + 3] = x.w;
  }
  uint32_t sg[4] = {0u, 0u, 0u, 0u};
  if (VS) {
    const uint4 x = *(const uint4*)(stg + Lo.sg_off + t * 16);
    sg[0] = x.x;
    sg[1] = x.y;
    sg[2] = x.z;
    sg[3] = x.w;
  }
#pragma unroll
  for (int g = 0; g < 4; ++g) {
#pragma unroll
    for (int P = 0; P < NP; ++P) {
      // the Walsh planes of a 1- or 2-bit codebook are its bit planes
      const uint32_t w = (VS && P == NP - 1) ? sg[g] : vw[g * BV + (P < BV ? P : 0)];
      uint8_t* row = avb + P * Lo.av_bytes;
      *(uint4*)(row + voff[2 * g]) = make_uint4(w & 0x01010101u, w & 0x02020202u, w & 0x04040404u, w & 0x08080808u);
      *(uint4*)(row + voff[2 * g + 1]) = make_uint4(w & 0x10101010u, w & 0x20202020u, w & 0x40404040u, w & 0x80808080u);
    }
  }
}

// HG: query heads per KV head (4 or 8, Hg <= HG); BK: key codebook bits; BV: value codebook bits;
// VS: value sign plane (Algorithm 2 values); KS: key sign plane (Algorithm 2 keys, BK <= 2)
// Register cap: the most that fits the warps an SM sub-partition holds (16384 registers each, 5 of
// the 19 warps, in units of 8 registers a thread).
template <int HG, int BK, int BV, int VS, int KS>
__global__ void __maxnreg__(96) attend_main_kernel(const __grid_constant__ AttParams p) {
  static_assert(att_warps(HG) == 19, "the register cap assumes 19 warps");
  constexpr bool SPLITV = att_split_v(HG);
  constexpr int NG = att_groups(HG);             // softmax groups
  constexpr int W_EXP = 2 + 4 * NG;              // first key expander warp
  constexpr int W_ACC = W_EXP + 4;               // first accumulator warp
  constexpr int W_VMMA = W_ACC + 4;              // value MMA warp (then the value expanders)
  constexpr int MK = walsh_count(BK);
  constexpr int MKT = MK + KS;                   // key operand planes (Walsh planes, sign plane)
  constexpr int MV = walsh_count(BV);
  static_assert(MKT <= 4, "key planes exceed the TMEM budget");
  constexpr uint32_t kAK0 = 0, AKS = 32 * MKT;   // key operand buffers [2][AKS columns]
  constexpr uint32_t kDS0 = 2 * AKS;             // scores [2][NQS]
  constexpr int NP = MV + VS;
  constexpr int NQ = HG <= 4 ? 16 : 32;
  constexpr int NQS = NQ * (1 + KS);            // score columns: Walsh part, then (KS) sign part
  constexpr int KSTEPS = MK * 128 / 32;          // K steps of the Walsh planes (the sign plane adds 4)
  // The chunk's fp16 norms ride with the key planes through TMEM (the key expanders store them, the
  // softmax warps load them with the scores): 4 buffers of 2 columns after the value products,
  // where they fit; else the softmax warps read them from the stage.
  constexpr uint32_t kNR0 = 2 * 32 * MKT + 2 * NQS + 2 * (MV + VS) * NQ;
  constexpr bool NT = kNR0 + 8 <= 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int nst = p.nst;
  const AttLayout Lo = att_layout(p, nst);
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
  const int64_t T = p.T, TS = p.tstride;
  const uint32_t dv0 = kDS0 + 2 * NQS;
  const uint32_t dv_cols = NP * NQ;
  // tokens in the last chunk of every slice (all other chunks are full)
  const int tail = (int)(T - (int64_t)(p.nchunk - 1) * kChunk);

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&bar[ST_FULL + s], 1);
      mbar_init(&bar[ST_EMPTY + s], (SPLITV ? 8 : 4) + (NT ? 0 : 4 * NG));   // key (and value) expanders, softmax
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[BQ_FULL + s], 1);
      mbar_init(&bar[BQ_EMPTY + s], 1);
      mbar_init(&bar[AK_FULL + s], 4);
      mbar_init(&bar[SC_DONE + s], 1);
      mbar_init(&bar[BW_FULL + s], 4 * NG);
      mbar_init(&bar[RUN_DONE + s], 2);
      mbar_init(&bar[RUN_FREE + s], 4);
      mbar_init(&bar[SC_FREE + s], 4 * NG);
    }
    for (int s = 0; s < 3; ++s) mbar_init(&bar[AV_FULL + s], 4);
    for (int s = 0; s < 6; ++s) mbar_init(&bar[V_DONE + s], 1);
    *abort_flag = 0;
    for (int s = 0; s < 4; ++s) ((int*)(scal + s * 64))[40] = ((int*)(scal + s * 64))[41] = -1;   // no chunk yet
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched as a dependent of the prep kernel: its query images, constants (and appended records)
  // are read only after this; the combine kernel may in turn be scheduled from here on
  grid_dep_wait();
  grid_dep_launch();
  const uint32_t tbase = *tmem_slot;

  ChunkIter it;
  it.init(p, c_begin);

  if (warp == 0) {
    // ------------------------------------ producer -------------------------------------------------
    // warp-uniform schedule; one elected lane issues the copies
    const uint32_t nb = (uint32_t)(NQ * MKT * d);
    RingPos rs{0, nst, 0u};
    for (int c = 0; c < nmy; ++c, it.next(), rs.next()) {
      if (c == 0 || it.cis == 0) {
        const int sg = it.seg;
        if (!mbar_wait_warp(&bar[BQ_EMPTY + (sg & 1)], ((sg >> 1) & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) break;
        if (elect_one_sync()) {
          mbar_arrive_expect_tx(&bar[BQ_FULL + (sg & 1)], nb);
          bulk_g2s(smem + Lo.off_bq + (sg & 1) * Lo.bq_bytes, p.bq_img + (size_t)it.slice * nb, nb,
                   &bar[BQ_FULL + (sg & 1)]);
        }
        __syncwarp();
      }
      const int st = rs.slot;
      if (!mbar_wait_warp(&bar[ST_EMPTY + st], rs.par ^ 1u, p.err, kDevTimeoutSync, abort_flag)) break;
      const int tc = it.cis == p.nchunk - 1 ? tail : kChunk;
      const int64_t vec0 = (int64_t)it.cs * TS + (int64_t)it.cis * kChunk;  // record of the first token
      const uint32_t kb = (uint32_t)tc * G * BK * 4;
      const uint32_t vb = (uint32_t)tc * G * BV * 4;
      const uint32_t sb = VS ? (uint32_t)tc * G * 4 : 0u;
      const uint32_t kgb = KS ? (uint32_t)tc * G * 4 : 0u;
      // norms of the first tc & ~7 tokens (whole 16-byte pieces; a ragged remainder is read by the
      // softmax warps themselves)
      const uint32_t nb2 = p.norm_bulk ? (uint32_t)(tc & ~7) * 2u : 0u;
      const uint32_t nrmb = nb2 * (2u + (VS ? 1u : 0u) + (KS ? 1u : 0u));
      uint8_t* stg = smem + Lo.off_stage + st * Lo.stage_bytes;
      if (elect_one_sync()) {
        mbar_arrive_expect_tx(&bar[ST_FULL + st], kb + vb + sb + kgb + nrmb);
        if (nb2) {
          uint8_t* sn = stg + Lo.nrm_off;
          bulk_g2s(sn, p.k_norms + vec0, nb2, &bar[ST_FULL + st]);
          bulk_g2s(sn + 2 * kChunk, p.v_norms + vec0, nb2, &bar[ST_FULL + st]);
          if (VS) bulk_g2s(sn + 4 * kChunk, p.v_gammas + vec0, nb2, &bar[ST_FULL + st]);
          if (KS) bulk_g2s(sn + 6 * kChunk, p.k_gammas + vec0, nb2, &bar[ST_FULL + st]);
        }
        bulk_g2s(stg, p.k_codes + vec0 * G * BK, kb, &bar[ST_FULL + st]);
        bulk_g2s(stg + Lo.kc_bytes, p.v_codes + vec0 * G * BV, vb, &bar[ST_FULL + st]);
        if (VS) bulk_g2s(stg + Lo.sg_off, p.v_signs + vec0 * G, sb, &bar[ST_FULL + st]);
        if (KS) bulk_g2s(stg + Lo.ks_off, p.k_signs + vec0 * G, kgb, &bar[ST_FULL + st]);
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    // ------------------------------------ key MMA issuer ------------------------------------------
    // The whole warp walks the schedule (its values are warp-uniform and stay in uniform
    // registers); one elected lane issues each group of tcgen05 instructions and their commits.
    const uint32_t id_s = idesc_i8_s32(128, NQ, false, true, false, false);
    // descriptor at the start of the query images; offsets below are added in 16-byte units
    const uint64_t dq0 = desc_kmajor_sw128(smem_u32(smem + Lo.off_bq));
    for (int c = 0; c < nmy; ++c, it.next()) {
      const int b = c & 1;
      const int sg = it.seg;
      if (c == 0 || it.cis == 0) {
        if (!mbar_wait_warp(&bar[BQ_FULL + (sg & 1)], (sg >> 1) & 1, p.err, kDevTimeoutLoad, abort_flag)) break;
      }
      if (!mbar_wait_warp(&bar[AK_FULL + b], (c >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
      // the scores buffer b is free once the softmax warps finished chunk c-2 (the whole chunk: the
      // key expanders of chunk c+2, which follow these MMAs, reuse the norm columns of chunk c-2)
      if (c >= 2 && !mbar_wait_warp(&bar[BW_FULL + b], ((c - 2) >> 1) & 1, p.err, kDevTimeoutSync, abort_flag))
        break;
      tc_fence_after();
      const uint64_t dq = dq0 + (((sg & 1) * Lo.bq_bytes) >> 4);
      const uint32_t ak = tbase + kAK0 + b * AKS;
      const uint32_t ds = tbase + kDS0 + b * NQS;
      const bool last = c == nmy - 1 || it.cis == p.nchunk - 1;
      if (elect_one_sync()) {
#pragma unroll
        for (int ks = 0; ks < KSTEPS + 4 * KS; ++ks) {
          // the sign plane's steps (ks >= KSTEPS) accumulate into their own columns
          const uint32_t kbyte = ks * 32, blk = kbyte >> 7, inb = kbyte & 127;
          const bool sgn = ks >= KSTEPS;
          mma_i8_ts(ds + (sgn ? NQ : 0), ak + ks * 8, dq + ((blk * NQ * 128 + inb) >> 4), id_s,
                    sgn ? ks > KSTEPS : ks > 0);
        }
        mma_commit(&bar[SC_DONE + b]);
        if (last) mma_commit(&bar[BQ_EMPTY + (sg & 1)]);
      }
      __syncwarp();
    }
  } else if (warp < W_EXP) {
    // ------------------------------------ softmax warps (thread = token) ---------------------------
    // group gq of four warps owns query heads [h0, h0 + HH); with two groups both track the same
    // value-norm maxima (same tokens, same rule), so the fixed-point scales agree
    constexpr int HH = HG / NG;
    const int q = warp & 3;
    const int gq = (warp - 2) >> 2;
    const int h0 = gq * HH;
    const int t = q * 32 + lane;                    // token inside the chunk == TMEM lane
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int Hg = p.Hg;
    float* rgrp = red + gq * 64;
    float mrun[HH], ha[HH], hb[HH], hs[HH], hq[HH];
    int hlim[HH];                                   // each head sees the slice's tokens t < hlim (causal)
    float vmax_run = 0.0f, gmax_run = 0.0f, sw = 1.0f, sw2 = 1.0f, isw = 1.0f, isw2 = 1.0f;
    bool ok = true;
    // this thread's token's share of the segment's sum of p (rescaled with the running maximum),
    // reduced over the group once, at the segment's end, into one of 4 slots (a slot is written again
    // four segments later, after the value MMA warp has read it)
    float lt[HH];
    float* segl = (float*)(smem + Lo.off_sum);      // [slot][warp][head]
    RingPos rs{0, nst, 0u};
    for (int c = 0; c < nmy; ++c, it.next(), rs.next()) {     // no early exit: the named barriers must match
      const int b = c & 1;
      const int tc = it.cis == p.nchunk - 1 ? tail : kChunk;
      const bool live = t < tc;
      uint16_t nk_n = 0, nv_n = 0, gm_n = 0, gk_n = 0;
      // fp16 norms of the chunk's tokens: with the scores (TMEM), else from the stage (bulk-copied
      // with the codes) where possible, else from global memory (dead tokens read as zero)
      if (!NT) ok = mbar_wait_warp(&bar[ST_FULL + rs.slot], rs.par, p.err, kDevTimeoutLoad, abort_flag) && ok;
      if (NT) {
      } else if (p.norm_bulk && t < (tc & ~7)) {
        const uint16_t* sn = (const uint16_t*)(smem + Lo.off_stage + rs.slot * Lo.stage_bytes + Lo.nrm_off);
        nk_n = sn[t];
        nv_n = sn[kChunk + t];
        if (VS) gm_n = sn[2 * kChunk + t];
        if (KS) gk_n = sn[3 * kChunk + t];
      } else if (live) {
        const int64_t rec = (int64_t)it.cs * TS + (int64_t)it.cis * kChunk + t;
        nk_n = __ldg(p.k_norms + rec);
        nv_n = __ldg(p.v_norms + rec);
        if (VS) gm_n = __ldg(p.v_gammas + rec);
        if (KS) gk_n = __ldg(p.k_gammas + rec);
      }
      if (!NT) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[ST_EMPTY + rs.slot]);   // done with the stage
      }
      if (c == 0 || it.cis == 0) {
        vmax_run = gmax_run = 0.0f;
        const float4* hc = (const float4*)(p.head_c + it.slice * 32);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          mrun[i] = -INFINITY;
          lt[i] = 0.0f;
          const float4 x = h0 + i < Hg ? __ldg(hc + h0 + i) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          ha[i] = -2.0f * x.x * p.scale_log2e;
          hb[i] = x.y * p.scale_log2e;
          // key sign term alpha gamma <q'', 2z - 1> = alpha gamma (2 2^-F'' D_z - Q'')
          hs[i] = 2.0f * p.alpha * x.z * p.scale_log2e;
          hq[i] = -p.alpha * x.w * p.scale_log2e;
          // virtual head h0 + i is query token j = pass * nqry + (h0 + i) / Hgr; tokens t < tlim0 + j
          const int j = (it.slice / p.cslices) * p.nqry + (h0 + i) / p.Hgr;
          hlim[i] = (h0 + i < Hg && j < p.nqtot) ? (int)(p.tlim0 + j) : 0;   // heads past Hg see nothing
        }
      }
      const int tg = it.cis * kChunk + t;           // this thread's token, counted in the slice
      ok = mbar_wait_warp(&bar[SC_DONE + b], (c >> 1) & 1, p.err, kDevTimeoutMma, abort_flag) && ok;
      tc_fence_after();
      uint32_t dsr[4 * HH], dzr[KS ? 4 * HH : 1];
      const uint32_t scol = tbase + lane_base + kDS0 + b * NQS + 4 * h0;
      if (HH == 2) tmem_ld8(scol, *(uint32_t(*)[8]) & dsr[0]);
      else tmem_ld16(scol, *(uint32_t(*)[16]) & dsr[0]);
      if (KS) {
        if (HH == 2) tmem_ld8(scol + NQ, *(uint32_t(*)[8]) & dzr[0]);
        else tmem_ld16(scol + NQ, *(uint32_t(*)[16]) & dzr[0]);
      }
      uint32_t nrw[2];
      if (NT) tmem_ld2(tbase + lane_base + kNR0 + (c & 3) * 2, nrw);
      tmem_ld_wait();
      if (NT) {
        nk_n = (uint16_t)(nrw[0] & 0xFFFFu);
        nv_n = (uint16_t)(nrw[0] >> 16);
        gm_n = (uint16_t)(nrw[1] & 0xFFFFu);
        gk_n = (uint16_t)(nrw[1] >> 16);
      }
      const float nk = __half2float(__ushort_as_half(nk_n)), nv = __half2float(__ushort_as_half(nv_n));
      const float gm = VS ? __half2float(__ushort_as_half(gm_n)) : 0.0f;
      const float gk = KS ? __half2float(__ushort_as_half(gk_n)) : 0.0f;
      tc_fence_before();
      float lg[HH];
      bool up = nv > vmax_run || nv * gm > gmax_run;
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        // the four limb products are exact integers below 2^21 in magnitude: pairs of limbs combine
        // exactly in 32 bits, then one fp32 rounding each
        const float dot = limbs_to_float(dsr[4 * i], dsr[4 * i + 1], dsr[4 * i + 2], dsr[4 * i + 3]);
        float sc = fmaf(ha[i], dot, hb[i]);
        if (KS) {
          const float dz = limbs_to_float(dzr[4 * i], dzr[4 * i + 1], dzr[4 * i + 2], dzr[4 * i + 3]);
          sc = fmaf(gk, fmaf(hs[i], dz, hq[i]), sc);
        }
        lg[i] = (live && tg < hlim[i]) ? nk * sc : -INFINITY;
        up = up || lg[i] > mrun[i];
      }
      float corr[HH];
#pragma unroll
      for (int i = 0; i < HH; ++i) corr[i] = 1.0f;
      bool changed = false;                         // a running maximum or a fixed-point scale moved
      if (bar_red_or(1 + 2 * gq, 128, up)) {
        // some token raised a running maximum: exchange the chunk maxima of the group's warps
        float* rb = rgrp + q * 16;
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float v = warp_max(lg[i]);
          if (lane == 0) rb[i] = v;
        }
        const float vm = warp_max(nv), gmx = warp_max(nv * gm);
        if (lane == 0) {
          rb[8] = vm;
          rb[9] = gmx;
        }
        bar_sync_named(2 + 2 * gq, 128);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float cm = fmaxf(fmaxf(rgrp[i], rgrp[16 + i]), fmaxf(rgrp[32 + i], rgrp[48 + i]));
          const float mn = fmaxf(mrun[i], cm);
          corr[i] = (mn == -INFINITY) ? 1.0f : fast_exp2(mrun[i] - mn);
          changed = changed || mn != mrun[i];
          mrun[i] = mn;
        }
        vmax_run = fmaxf(vmax_run, fmaxf(fmaxf(rgrp[8], rgrp[24]), fmaxf(rgrp[40], rgrp[56])));
        gmax_run = fmaxf(gmax_run, fmaxf(fmaxf(rgrp[9], rgrp[25]), fmaxf(rgrp[41], rgrp[57])));
        int E1 = 0, E2 = 0;
        frexpf(fmaxf(vmax_run, 1e-30f), &E1);
        frexpf(fmaxf(gmax_run, 1e-30f), &E2);
        E1 = max(E1, -80);
        E2 = max(E2, -80);
        const float nisw = ldexpf(1.0f, E1 - 23), nisw2 = ldexpf(1.0f, E2 - 23);
        changed = changed || nisw != isw || nisw2 != isw2;
        sw = ldexpf(1.0f, 23 - E1);                // w * sw <= 2^23 for every w <= vmax_run
        sw2 = ldexpf(1.0f, 23 - E2);               // likewise for w * gamma
        isw = nisw;
        isw2 = nisw2;
      }
      // weights: p = 2^(lg - m) <= 1, w = p |v|, w' = w gamma, as 24-bit unsigned fixed point
      uint32_t wv[HH], wz[HH];
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        const float pr = (lg[i] == -INFINITY) ? 0.0f : fast_exp2(lg[i] - mrun[i]);
        const float w = pr * nv;
        wv[i] = fixed24(w, sw);
        wz[i] = VS ? fixed24(w * gm, sw2) : 0u;
        lt[i] = fmaf(lt[i], corr[i], pr);
      }
      if (c >= 2)
        ok = mbar_wait_warp(&bar[V_DONE + (c - 2) % 6], ((c - 2) / 6) & 1, p.err, kDevTimeoutMma, abort_flag) && ok;
      if (c == nmy - 1 || it.cis == p.nchunk - 1) {
        // the segment ends with this chunk: the group's sums of p of its heads
        float* lp = segl + ((it.seg & 3) * 4 + q) * 8;
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          float sl = lt[i];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, o);
          if (lane == 0) lp[h0 + i] = sl;
        }
      }
      // this group's heads fill 4 HH bytes of the token's row (block h0 / 4, byte 4 (h0 % 4))
      uint8_t* bwb = smem + Lo.off_bw + b * Lo.bw_buf + (h0 >> 2) * kChunk * 16 + t * 16 + (h0 & 3) * 4;
      if (HH == 2) {
        *(uint2*)bwb = make_uint2(wv[0], wv[HH > 1 ? 1 : 0]);
        if (VS) *(uint2*)(bwb + Lo.bw_kind) = make_uint2(wz[0], wz[HH > 1 ? 1 : 0]);
      } else {
        *(uint4*)bwb = make_uint4(wv[0], wv[HH > 1 ? 1 : 0], wv[HH > 2 ? 2 : 0], wv[HH > 3 ? 3 : 0]);
        if (VS)
          *(uint4*)(bwb + Lo.bw_kind) = make_uint4(wz[0], wz[HH > 1 ? 1 : 0], wz[HH > 2 ? 2 : 0], wz[HH > 3 ? 3 : 0]);
      }
      fence_proxy_async_smem();
      if (q == 0 && lane == 0 && (changed || c == 0 || it.cis == 0)) {
        // where this group's maxima or scales moved (or a segment starts), the chunk starts a new run:
        // its scalars for the value MMA warp (4-deep ring), stamped with the chunk
        float* sc = scal + (c & 3) * 64;
#pragma unroll
        for (int i = 0; i < HH; ++i) sc[16 + h0 + i] = mrun[i];
        sc[32 + 2 * gq] = isw;
        sc[33 + 2 * gq] = isw2;
        ((int*)sc)[40 + gq] = c;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[BW_FULL + b]);
    }
    (void)ok;
  } else if (warp < W_ACC) {
    // ------------------------------------ expanders (thread = token) -------------------------------
    const int q = warp & 3;
    const int t = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    uint32_t voff[8];                               // this token's 16-byte slots in a value plane
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      voff[2 * g] = sw128_offset(t, g * 32, 128);
      voff[2 * g + 1] = sw128_offset(t, g * 32 + 16, 128);
    }
    RingPos rs{0, nst, 0u};
    for (int c = 0; c < nmy; ++c, rs.next(), it.next()) {
      const int st = rs.slot, b = c & 1;
      if (!mbar_wait_warp(&bar[ST_FULL + st], rs.par, p.err, kDevTimeoutLoad, abort_flag)) break;
      if (c >= 2 && !mbar_wait_warp(&bar[SC_DONE + b], ((c - 2) >> 1) & 1, p.err, kDevTimeoutMma, abort_flag))
        break;
      tc_fence_after();
      const uint8_t* stg = smem + Lo.off_stage + st * Lo.stage_bytes;
      // keys: the token's 4 x BK plane words -> MK Walsh planes of expanded bytes in TMEM
      uint32_t kw[4 * BK];
#pragma unroll
      for (int v4 = 0; v4 < BK; ++v4) {
        const uint4 x = *(const uint4*)(stg + t * 16 * BK + v4 * 16);
        kw[4 * v4] = x.x;
        kw[4 * v4 + 1] = x.y;
        kw[4 * v4 + 2] = x.z;
        kw[4 * v4 + 3] = x.w;
      }
      const uint32_t ak = tbase + lane_base + kAK0 + b * AKS;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
#pragma unroll
        for (int S = 0; S < MK; ++S) {
          const int m = walsh_mask(BK, S);
          uint32_t w = 0;
          if (m & 1) w ^= kw[g * BK];
          if (BK > 1 && (m & 2)) w ^= kw[g * BK + (BK > 1 ? 1 : 0)];
          if (BK > 2 && (m & 4)) w ^= kw[g * BK + (BK > 2 ? 2 : 0)];
          uint32_t r[8];
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) r[s8] = w & (0x01010101u << s8);
          tmem_st8(ak + S * 32 + g * 8, r);
        }
      }
      if (KS) {
        // the key sign plane z (Algorithm 2 keys) after the Walsh planes
        const uint4 x = *(const uint4*)(stg + Lo.ks_off + t * 16);
        const uint32_t zw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t r[8];
#pragma unroll
          for (int s8 = 0; s8 < 8; ++s8) r[s8] = zw[g] & (0x01010101u << s8);
          tmem_st8(ak + MK * 32 + g * 8, r);
        }
      }
      if (NT) {
        // the token's fp16 norms for the softmax warps: (key norm | value norm << 16), (value gamma |
        // key gamma << 16), in buffer c % 4 (free: the key MMAs of chunk c-2, which this warp waited
        // for, followed the softmax of chunk c-4)
        const int tc = it.cis == p.nchunk - 1 ? tail : kChunk;
        uint32_t nr[2] = {0u, 0u};
        if (p.norm_bulk && t < (tc & ~7)) {
          const uint16_t* sn = (const uint16_t*)(stg + Lo.nrm_off);
          nr[0] = (uint32_t)sn[t] | ((uint32_t)sn[kChunk + t] << 16);
          nr[1] = (VS ? (uint32_t)sn[2 * kChunk + t] : 0u) | (KS ? (uint32_t)sn[3 * kChunk + t] << 16 : 0u);
        } else if (t < tc) {
          const int64_t rec = (int64_t)it.cs * TS + (int64_t)it.cis * kChunk + t;
          nr[0] = (uint32_t)__ldg(p.k_norms + rec) | ((uint32_t)__ldg(p.v_norms + rec) << 16);
          nr[1] = (VS ? (uint32_t)__ldg(p.v_gammas + rec) : 0u) | (KS ? (uint32_t)__ldg(p.k_gammas + rec) << 16 : 0u);
        }
        tmem_st2(tbase + lane_base + kNR0 + (c & 3) * 2, nr);
      }
      // the key planes (and norms) are complete once this warp's TMEM stores are
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[AK_FULL + b]);
      if (SPLITV) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[ST_EMPTY + st]);
        continue;
      }
      // values: plane words (and sign words) -> expanded bytes, one token row per plane; the
      // planes of chunk c - 3 (same buffer) must have been consumed
      const int c3 = c % 3;
      if (c >= 3 && !mbar_wait_warp(&bar[V_DONE + (c - 3) % 6], ((c - 3) / 6) & 1, p.err, kDevTimeoutMma, abort_flag))
        break;
      expand_v_rows<BV, VS, NP>(p, Lo, stg, smem + Lo.off_av + c3 * NP * Lo.av_bytes, t, voff);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[AV_FULL + c3]);
        mbar_arrive(&bar[ST_EMPTY + st]);
      }
    }
  } else if (warp < W_VMMA) {
    // ------------------------------------ accumulators (thread = coordinate row) -------------------
    // One pass per run: the run's limb sums from TMEM and its exact weight sums are folded in int64,
    //   O_P = 2^s W - 2 Y_P (Walsh planes),  O_z = 2 Y_z - 2^s W' (sign plane),
    // then added to the running state with the rescale from the previous run's maxima.
    const int q = warp & 3;
    const int m = q * 32 + lane;                 // TMEM lane = M index of the value MMA
    const int g = m >> 5, r = m & 31, s = r >> 2, jj = r & 3;
    const int coord = 32 * g + 8 * jj + s;       // coordinate this row holds
    const float rowscale = ldexpf(1.0f, -s);
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int Hg = p.Hg;
    float acc[NP][HG];                           // folded planes O_P per head
    float Lr[HG];                                // sum of p
    float macc[HG];                              // maxima the state refers to
    bool fresh = true;                           // the next run starts a segment
    for (int R = 0; nmy > 0; ++R) {
      const int nb = R & 1;
      if (!mbar_wait_warp(&bar[RUN_DONE + nb], (R >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      const uint32_t col = tbase + lane_base + dv0 + nb * dv_cols;
      const uint8_t* rr = smem + Lo.off_run + nb * kRunRec;
      const float* rm = (const float*)rr;
      const unsigned long long* rs = (const unsigned long long*)(rr + 64);
      const int flags = *(const int*)(rr + 40);
      const int seg = *(const int*)(rr + 44);
      const int sgs = *(const int*)(rr + 48);
      const float fw = rm[8] * rowscale, fz = rm[9] * rowscale;
      if (fresh) {
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          Lr[h] = 0.0f;
          macc[h] = -INFINITY;
#pragma unroll
          for (int P = 0; P < NP; ++P) acc[P][h] = 0.0f;
        }
      }
      float corr[HG];
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const float mr = rm[h];
        corr[h] = macc[h] == -INFINITY ? 0.0f : fast_exp2(macc[h] - mr);
        macc[h] = mr;
        // sum of p of the segment (at the segment's final maxima), with its last run
        if ((flags & 1) && m == 0) Lr[h] = ((const float*)(rr + 192))[h];
      }
      // one plane at a time (keeps the TMEM columns of a single plane in registers)
#pragma unroll
      for (int P = 0; P < NP; ++P) {
        const bool sgn = VS && P == NP - 1;
        uint32_t dv[NQ];
        tmem_ld16(col + P * NQ, *(uint32_t(*)[16]) & dv[0]);
        if (NQ > 16) tmem_ld16(col + P * NQ + 16, *(uint32_t(*)[16]) & dv[NQ > 16 ? 16 : 0]);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          // Y = sum over the run of 2^s b w (three 8-bit limb columns), exact in int64
          const long long y = (long long)dv[4 * h] + ((long long)dv[4 * h + 1] << 8) + ((long long)dv[4 * h + 2] << 16);
          const long long o = sgn ? 2 * y - ((long long)rs[8 + h] << s) : ((long long)rs[h] << s) - 2 * y;
          acc[P][h] = fmaf(acc[P][h], corr[h], (float)o * (sgn ? fz : fw));
        }
      }
      // the buffer and the record may now be reused by the run after next
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[RUN_FREE + nb]);
      fresh = (flags & 1) != 0;
      if (fresh) {
        // the last run of a segment: write the segment's partial state
        float* rec = p.partial + ((size_t)sgs * p.maxseg + seg) * Hg * att_rec(d);
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          if (h < Hg) {
            float* rh = rec + h * att_rec(d);
#pragma unroll
            for (int P = 0; P < NP; ++P) rh[4 + P * d + coord] = acc[P][h];
            if (m == 0) {
              rh[0] = macc[h];
              rh[1] = Lr[h];
              rh[2] = 1.0f;
              rh[3] = 0.0f;
            }
          }
        }
      }
      if (flags & 2) break;
    }
  } else if (warp == W_VMMA) {
    // ------------------------------------ value MMA issuer ------------------------------------------
    // Runs beside the key MMA warp so that neither warp's barrier waits and commits sit behind the
    // other's tensor-core work. Warp-uniform schedule, one elected lane issues. It also keeps the
    // runs: a chunk whose softmax scalars moved starts a new run in the other TMEM buffer. The warp
    // also adds up each run's weights exactly (lane = four tokens of each chunk) from the weight tiles.
    const uint32_t id_v = idesc_i8_s32(128, NQ, false, false, true, true);
    const uint64_t da0 = desc_smem(smem_u32(smem + Lo.off_av), 1024, 1024, 2);
    const uint64_t db0 = desc_smem(smem_u32(smem + Lo.off_bw), 128, kChunk * 16, 0);
    int R = -1, runlen = 0;
    bool open = false;
    float cur_sc = 0.0f;                         // lane < 10: scalar `lane` of the current run
    // this lane's share of the run's weight sums (tokens lane + 32 j of every chunk; below 2^33)
    unsigned long long aw[HG], az[VS ? HG : 1];
    const float* segl = (const float*)(smem + Lo.off_sum);
    auto close_run = [&](int flags, int seg) {
      uint8_t* rr = smem + Lo.off_run + (R & 1) * kRunRec;
      unsigned long long* rs = (unsigned long long*)(rr + 64);
#pragma unroll
      for (int h = 0; h < HG; ++h) {
        const unsigned long long tw = warp_sum_u64(aw[h]);
        const unsigned long long tz = VS ? warp_sum_u64(az[VS ? h : 0]) : 0ull;
        if (lane == 0) {
          rs[h] = tw;
          rs[8 + h] = tz;
        }
      }
      if ((flags & 1) && lane < 8) {
        // the segment's sums of p (four warp partials per head)
        const float* lp = segl + (it.seg & 3) * 32 + lane;
        ((float*)(rr + 192))[lane] = (lp[0] + lp[8]) + (lp[16] + lp[24]);
      }
      if (lane == 0) {
        *(int*)(rr + 40) = flags;
        *(int*)(rr + 44) = seg;
      }
      __syncwarp();
      if (elect_one_sync()) {
        mma_commit(&bar[RUN_DONE + (R & 1)]);     // the run's MMAs are complete
        mbar_arrive(&bar[RUN_DONE + (R & 1)]);    // and its record is written
      }
      __syncwarp();
      open = false;
    };
    for (int c = 0; c < nmy; ++c, it.next()) {
      const int b = c & 1, c3 = c % 3;
      if (!mbar_wait_warp(&bar[BW_FULL + b], (c >> 1) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
      if (!mbar_wait_warp(&bar[AV_FULL + c3], (c / 3) & 1, p.err, kDevTimeoutSync, abort_flag)) break;
      const float* sc = scal + (c & 3) * 64;
      const bool st0 = ((const int*)sc)[40] == c, st1 = NG > 1 && ((const int*)sc)[41] == c;
      const bool newrun = !open || st0 || st1 || runlen == kMaxRun;
      if (newrun) {
        if (open) close_run(0, 0);
        ++R;
        runlen = 0;
#pragma unroll
        for (int h = 0; h < HG; ++h) {
          aw[h] = 0;
          if (VS) az[VS ? h : 0] = 0;
        }
        // the other buffer's previous run must have been drained by the accumulators
        if (R >= 2 && !mbar_wait_warp(&bar[RUN_FREE + (R & 1)], ((R >> 1) - 1) & 1, p.err, kDevTimeoutSync, abort_flag))
          break;
        uint8_t* rr = smem + Lo.off_run + (R & 1) * kRunRec;
        // lanes 0..9 keep the run's scalars (8 maxima, 1/sw, 1/sw'), from the stamped groups
        if (lane < 8) {
          if ((lane / (HG / NG) == 0 ? st0 : st1)) cur_sc = sc[16 + lane];
        } else if (lane < 10) {
          if (st0 || st1) cur_sc = sc[32 + (st0 ? 0 : 2) + lane - 8];
        }
        if (lane < 10) ((float*)rr)[lane] = cur_sc;
        if (lane == 10) *(int*)(rr + 48) = it.slice;
        open = true;
      }
      tc_fence_after();
      const uint32_t dcol = tbase + dv0 + (R & 1) * dv_cols;
      const uint64_t da = da0 + ((c3 * NP * Lo.av_bytes) >> 4);
      const uint64_t db = db0 + ((b * Lo.bw_buf) >> 4);
      if (elect_one_sync()) {
#pragma unroll
        for (int P = 0; P < NP; ++P) {
          const bool sgn = VS && P == NP - 1;
#pragma unroll
          for (int ks = 0; ks < kChunk / 32; ++ks)
            mma_i8_ss(dcol + P * NQ, da + ((P * Lo.av_bytes + ks * 32 * 128) >> 4),
                      db + (((sgn ? Lo.bw_kind : 0u) + ks * 32 * 16) >> 4), id_v, (ks > 0 || !newrun) ? 1u : 0u);
        }
      }
      __syncwarp();
      {
        // the chunk's weights into the run sums, read before the commit below releases the tiles to
        // the softmax warps (the adds consume the loads first)
        const uint8_t* bwt = smem + Lo.off_bw + b * Lo.bw_buf + lane * 16;
#pragma unroll
        for (int blk = 0; blk < HG / 4; ++blk) {
#pragma unroll
          for (int kind = 0; kind < 1 + VS; ++kind) {
            const uint8_t* x = bwt + blk * kChunk * 16 + kind * Lo.bw_kind;
            const uint4 a0 = *(const uint4*)x, a1 = *(const uint4*)(x + 32 * 16);
            const uint4 a2 = *(const uint4*)(x + 64 * 16), a3 = *(const uint4*)(x + 96 * 16);
            const uint32_t s4[4] = {(a0.x + a1.x) + (a2.x + a3.x), (a0.y + a1.y) + (a2.y + a3.y),
                                    (a0.z + a1.z) + (a2.z + a3.z), (a0.w + a1.w) + (a2.w + a3.w)};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              if (kind == 0) aw[4 * blk + j] += s4[j];
              else az[VS ? 4 * blk + j : 0] += s4[j];
            }
          }
        }
      }
      __syncwarp();
      if (elect_one_sync()) mma_commit(&bar[V_DONE + c % 6]);
      __syncwarp();
      ++runlen;
      if (c == nmy - 1 || it.cis == p.nchunk - 1) {
        const int seg = (c_begin + c) / p.per_cta - (it.slice * p.nchunk) / p.per_cta;   // CTA ordinal in the slice
        close_run(1 | (c == nmy - 1 ? 2 : 0), seg);
      }
    }
  } else if (SPLITV) {
    // ------------------------------------ value expanders (last four warps, thread = token) -------
    const int q = warp & 3;
    const int t = q * 32 + lane;
    uint32_t voff[8];                               // this token's 16-byte slots in a value plane
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      voff[2 * g] = sw128_offset(t, g * 32, 128);
      voff[2 * g + 1] = sw128_offset(t, g * 32 + 16, 128);
    }
    RingPos rs{0, nst, 0u};
    for (int c = 0; c < nmy; ++c, rs.next()) {
      const int st = rs.slot, c3 = c % 3;
      if (!mbar_wait_warp(&bar[ST_FULL + st], rs.par, p.err, kDevTimeoutLoad, abort_flag)) break;
      // the planes of chunk c - 3 (same buffer) must have been consumed
      if (c >= 3 && !mbar_wait_warp(&bar[V_DONE + (c - 3) % 6], ((c - 3) / 6) & 1, p.err, kDevTimeoutMma, abort_flag))
        break;
      expand_v_rows<BV, VS, NP>(p, Lo, smem + Lo.off_stage + st * Lo.stage_bytes,
                                smem + Lo.off_av + c3 * NP * Lo.av_bytes, t, voff);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar[AV_FULL + c3]);
        mbar_arrive(&bar[ST_EMPTY + st]);
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
size_t combine_smem_bytes(int vsign) { return (size_t)(vsign ? 2 : 1) * 128 * 128 * sizeof(float); }

__global__ void attend_combine_kernel(const __grid_constant__ AttParams p) {
  const int slice = blockIdx.x;              // one block per work slice, all its virtual heads
  const int cs = slice % p.cslices, ps = slice / p.cslices;
  const int b = cs / p.Hkv, hk = cs % p.Hkv;
  const int d = p.d, i = threadIdx.x, Hg = p.Hg;
  extern __shared__ float cmb_mat[];         // Pi, then S (Algorithm 2 values): [128][128]
  __shared__ float orot[8][128], osgn[8][128];
  __shared__ float mmax[8], linv[8];
  // Pi (and S) into shared memory (coalesced 16-byte copies, all in flight at once); column j of
  // Pi^T is row j of Pi, read across the threads without bank conflicts
  for (int mtx = 0; mtx < (p.vsign ? 2 : 1); ++mtx) {
    const float4* src = (const float4*)(mtx ? p.S : p.Pi);
    float4* dst = (float4*)(cmb_mat + mtx * 128 * 128);
#pragma unroll 8
    for (int o = i; o < 128 * 32; o += 128) dst[o] = __ldg(src + o);
  }
  grid_dep_wait();                           // the main kernel's partial states
  // CTAs that touched this slice
  const int first = (slice * p.nchunk) / p.per_cta;
  const int last = (slice * p.nchunk + p.nchunk - 1) / p.per_cta;
  const int nseg = last - first + 1;
  const float* base0 = p.partial + (size_t)slice * p.maxseg * Hg * att_rec(d);
  const size_t stride = (size_t)Hg * att_rec(d);
  if (i < Hg) {
    const float* base = base0 + (size_t)i * att_rec(d);
    float M = -INFINITY;
    for (int sgi = 0; sgi < nseg; ++sgi) M = fmaxf(M, base[sgi * stride]);
    float L = 0.0f;
    for (int sgi = 0; sgi < nseg; ++sgi) {
      const float ms = base[sgi * stride];
      if (ms > -INFINITY) L += base[sgi * stride + 1] * exp2f(ms - M);
    }
    mmax[i] = M;
    linv[i] = L > 0.0f ? 1.0f / L : 0.0f;
  }
  __syncthreads();
  for (int h = 0; h < Hg; ++h) {
    const float* base = base0 + (size_t)h * att_rec(d);
    float y[3] = {0.0f, 0.0f, 0.0f};
    for (int sgi = 0; sgi < nseg; ++sgi) {
      const float ms = base[sgi * stride];
      if (ms == -INFINITY) continue;
      const float f = exp2f(ms - mmax[h]);
      for (int P = 0; P < p.np; ++P) y[P] = fmaf(base[sgi * stride + 4 + P * d + i], f, y[P]);
    }
    float a = 0.0f;
    for (int P = 0; P < p.mv; ++P) a = fmaf(p.beta_v[P], y[P], a);
    orot[h][i] = a * linv[h];
    osgn[h][i] = p.vsign ? y[p.np - 1] * linv[h] : 0.0f;
  }
  __syncthreads();
  // out_h[i] = sum_j Pi[j][i] orot_h[j] + alpha sum_j S[j][i] osgn_h[j]
  float acc[8], z[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) acc[h] = z[h] = 0.0f;
  const float* scol = cmb_mat + 128 * 128;
#pragma unroll 4
  for (int j = 0; j < 128; ++j) {
    const float pj = cmb_mat[j * 128 + i];
    const float sj = p.vsign ? scol[j * 128 + i] : 0.0f;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < Hg) {
        acc[h] = fmaf(pj, orot[h][j], acc[h]);
        if (p.vsign) z[h] = fmaf(sj, osgn[h][j], z[h]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h >= Hg) break;
    const int jq = ps * p.nqry + h / p.Hgr;
    if (jq >= p.nqtot) continue;               // a virtual head past the last query token
    const size_t ooff = (size_t)b * p.q_bs + (size_t)jq * p.q_js + (size_t)(hk * p.Hgr + h % p.Hgr) * d;
    p.out[ooff + i] = p.vsign ? fmaf(p.alpha, z[h], acc[h]) : acc[h];
  }
}

using MainKernel = void (*)(AttParams);

template <int HG, int BK, int KS>
MainKernel pick_v(int bv, int vs) {
  if (bv == 1) return vs ? attend_main_kernel<HG, BK, 1, 1, KS> : attend_main_kernel<HG, BK, 1, 0, KS>;
  return vs ? attend_main_kernel<HG, BK, 2, 1, KS> : attend_main_kernel<HG, BK, 2, 0, KS>;
}
template <int HG>
MainKernel pick_k(int bk, int bv, int vs, int ks) {
  if (ks) return bk == 1 ? pick_v<HG, 1, 1>(bv, vs) : pick_v<HG, 2, 1>(bv, vs);   // key codebooks <= 2 bits
  if (bk == 1) return pick_v<HG, 1, 0>(bv, vs);
  if (bk == 2) return pick_v<HG, 2, 0>(bv, vs);
  return pick_v<HG, 3, 0>(bv, vs);
}
MainKernel pick_main(int hg, int bk, int bv, int vs, int ks) {
  return hg <= 4 ? pick_k<4>(bk, bv, vs, ks) : pick_k<8>(bk, bv, vs, ks);
}

struct AttPlan {
  AttParams p;
  size_t bq_bytes, hc_bytes, part_bytes, total;
};

// Plan of one pass over T tokens of every slice with nqry query tokens per slice (Hg = nqry x Hq/Hkv
// virtual heads, at most 8).
bool att_plan(int B, int Hq, int Hkv, int64_t T, int d, int nsm, AttPlan& pl, int nqry = 1, int npass = 1) {
  AttParams& p = pl.p;
  p = AttParams{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Hgr = Hq / Hkv;
  p.nqry = nqry;
  p.Hg = nqry * p.Hgr;
  p.q_bs = (int64_t)Hq * d;
  p.q_js = 0;
  p.tlim0 = T;
  p.d = d;
  p.G = d / 32;
  p.T = T;
  p.tstride = T;
  p.cslices = B * Hkv;
  p.slices = npass * p.cslices;
  p.nqtot = nqry;
  p.nchunk = (int)((T + kChunk - 1) / kChunk);
  const long long totalc = (long long)p.slices * p.nchunk;
  const int ncta = (int)std::min<long long>(nsm, totalc);
  p.per_cta = (int)((totalc + ncta - 1) / ncta);
  p.maxseg = (p.nchunk + p.per_cta - 1) / p.per_cta + 1;
  p.nq = p.Hg <= 4 ? 16 : 32;      // the kernel is built for 4 or 8 (virtual) heads per KV head
  pl.bq_bytes = (size_t)p.slices * p.nq * 4 * d;       // mk <= 4
  pl.hc_bytes = (size_t)p.slices * 8 * 4 * sizeof(float);   // head_c [slices][8 heads][4]
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

namespace tq {
namespace {
// Geometry of one attention pass: nqry query tokens per slice, q / out strides, causal limit.
struct PassGeom {
  int nqry;                      // query tokens per cache slice and pass (1 for decode)
  int npass;                     // passes in the launch (query tokens nqry * npass >= nqtot)
  int nqtot;                     // query tokens in all
  int64_t q_bs, q_js;            // element strides of q / out: batch, query token
  int64_t tlim0;                 // query token j attends t < tlim0 + j
};

// The new token of every slice for tq_attend_append (written into slot t_new by the prep kernel).
struct AppendArgs {
  const void* k_new;
  const void* v_new;
  int x_dtype;
  int64_t t_new;
  uint32_t* k_codes;
  uint16_t* k_norms;
  uint32_t* v_codes;
  uint32_t* v_signs;
  uint16_t* v_norms;
  uint16_t* v_gammas;
};

// Argument checks shared by the attention entry points (no work is enqueued on failure).
tq_status attend_check(const std::string& f, const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                       int32_t Hkv, int64_t T, int64_t tstride, int32_t d, const void* q, int32_t q_dtype,
                       const void* rot, const uint32_t* k_codes, const uint16_t* k_norms, const uint32_t* k_signs,
                       const uint16_t* k_gammas, const uint32_t* v_codes, const uint32_t* v_signs,
                       const uint16_t* v_norms, const uint16_t* v_gammas, const float* out, const void* ws) {
  if (!cb_k || !cb_v || !q || !rot || !k_codes || !k_norms || !v_codes || !v_norms || !out || !ws)
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": NULL pointer");
  if ((v_signs == nullptr) != (v_gammas == nullptr))
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": v_signs and v_gammas must both be NULL or both be set");
  if ((k_signs == nullptr) != (k_gammas == nullptr))
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": k_signs and k_gammas must both be NULL or both be set");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || Hq % Hkv)
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": bad B / Hq / Hkv / T");
  if (tstride < T) return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": fewer cache slots than tokens");
  if (d != 128) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": this build supports d = 128");
  if (Hq / Hkv > 8) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": at most 8 query heads per KV head");
  if (T > ((int64_t)1 << 31)) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": T too large");
  if (cb_k->d != d || cb_v->d != d) return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": codebook d mismatch");
  if (cb_k->bits < 1 || cb_k->bits > 3)
    return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": key codebooks of 1..3 bits are supported");
  const bool ksign = k_signs != nullptr;
  if (ksign && cb_k->bits > 2)
    return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": Algorithm 2 keys need a key codebook of 1..2 bits");
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
  if (!aligned16(k_codes) || !aligned16(v_codes) || (vsign && !aligned16(v_signs)) || (ksign && !aligned16(k_signs)) ||
      !aligned16(ws) ||
      !aligned16(rot) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, std::string(f) + ": pointers must be 16-byte aligned");
  return TQ_OK;
}

// One pass: prep, main and combine kernels over the first T tokens of every slice.
tq_status attend_pass(const char* f, const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                      int32_t Hkv, int64_t T, int64_t tstride, int32_t d, const void* q, int32_t q_dtype,
                      const void* rot, const uint32_t* k_codes, const uint16_t* k_norms, const uint32_t* k_signs,
                      const uint16_t* k_gammas, const uint32_t* v_codes, const uint32_t* v_signs,
                      const uint16_t* v_norms, const uint16_t* v_gammas, float scale, float* out, void* ws,
                      size_t ws_bytes, void* stream, const PassGeom& g, const AppendArgs* app = nullptr) {
  const bool ksign = k_signs != nullptr;
  const bool vsign = v_signs != nullptr;
  AttPlan pl;
  att_plan(B, Hq, Hkv, T, d, sm_count(), pl, g.nqry, g.npass);
  if (ws_bytes < pl.total) return fail(TQ_ERR_WORKSPACE, std::string(f) + ": workspace too small");
  AttParams& p = pl.p;
  p.tstride = tstride;
  p.q_bs = g.q_bs;
  p.q_js = g.q_js;
  p.tlim0 = g.tlim0;
  p.nqtot = g.nqtot;
  int kmask[8], vmask[8];
  float kbeta[8], vbeta[8];
  p.bk = cb_k->bits;
  p.ksign = ksign ? 1 : 0;
  p.mk = walsh_planes(cb_k, kmask, kbeta);
  for (int i = 0; i < p.mk; ++i) p.beta_k[i] = kbeta[i];
  p.bv = cb_v->bits;
  p.mv = walsh_planes(cb_v, vmask, vbeta);
  for (int i = 0; i < p.mv; ++i) p.beta_v[i] = vbeta[i];
  p.vsign = vsign ? 1 : 0;
  p.np = p.mv + p.vsign;
  // scale <= 0 (or NaN) selects the plain attention scale 1/sqrt(d)
  if (!(scale > 0.0f)) scale = (float)(1.0 / std::sqrt((double)d));
  p.scale_log2e = scale * kLog2e;
  p.alpha = (float)(std::sqrt(M_PI / 2.0) / d);
  p.q = q;
  p.q_bf16 = q_dtype == TQ_BF16;
  RotLayout RL = rot_layout(d);
  p.Pi = (const float*)((const char*)rot + RL.pi32);
  p.S = (const float*)((const char*)rot + RL.s32);
  p.k_codes = k_codes;
  p.k_norms = k_norms;
  p.k_signs = k_signs;
  p.k_gammas = k_gammas;
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
  p.norm_bulk = (tstride % 8 == 0) && aligned16(k_norms) && aligned16(v_norms) && (!v_gammas || aligned16(v_gammas)) &&
                (!k_gammas || aligned16(k_gammas));
  if (app) {
    p.k_new = app->k_new;
    p.v_new = app->v_new;
    p.x_bf16 = app->x_dtype == TQ_BF16;
    p.t_new = app->t_new;
    p.kw_codes = app->k_codes;
    p.kw_norms = app->k_norms;
    p.vw_codes = app->v_codes;
    p.vw_signs = app->v_signs;
    p.vw_norms = app->v_norms;
    p.vw_gammas = app->v_gammas;
    for (int k = 0; k < 8; ++k) {
      p.ck[k] = k < cb_k->levels ? cb_k->c[k] : 0.0f;
      p.tk[k] = k < cb_k->levels - 1 ? cb_k->t[k] : 0.0f;
      p.cv[k] = k < cb_v->levels ? cb_v->c[k] : 0.0f;
      p.tv[k] = k < cb_v->levels - 1 ? cb_v->t[k] : 0.0f;
    }
  }
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, std::string(f) + ": no device error word");
  const AttLayout L0 = att_layout(p, 0);
  const int nst = (int)std::min<long long>(kMaxStages, ((long long)kMaxSmem - (long long)L0.total) / L0.stage_bytes);
  if (nst < 2) return fail(TQ_ERR_UNSUPPORTED, std::string(f) + ": shared memory too small for these bit widths");
  p.nst = nst;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  const size_t prep_sm = prep_smem_bytes(p.ksign), cmb_sm = combine_smem_bytes(p.vsign);
  e = cudaFuncSetAttribute(attend_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)prep_sm);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attend_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cmb_sm);
  if (e != cudaSuccess) return cuda_fail(e, (std::string(f) + ": shared memory attribute").c_str());
  attend_prep_kernel<<<p.slices, 128, prep_sm, st>>>(p);
  const AttLayout Lo = att_layout(p, nst);
  const MainKernel kern = pick_main(p.Hg, p.bk, p.bv, p.vsign, p.ksign);
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, (std::string(f) + ": shared memory attribute").c_str());
  const long long totalc = (long long)p.slices * p.nchunk;
  const int grid = (int)((totalc + p.per_cta - 1) / p.per_cta);
  // main and combine are launched as programmatic dependents of the kernel before them: their
  // launch and set-up overlap its tail, and each waits (griddepcontrol) before reading its results
  cudaLaunchAttribute dep[1];
  dep[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  dep[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(32 * att_warps(p.Hg <= 4 ? 4 : 8));
  cfg.dynamicSmemBytes = Lo.total;
  cfg.stream = st;
  cfg.attrs = dep;
  cfg.numAttrs = 1;
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, (std::string(f) + ": launch").c_str());
  if ((e = cudaLaunchKernelEx(&cfg, kern, p)) != cudaSuccess) return cuda_fail(e, (std::string(f) + ": launch").c_str());
  cfg.gridDim = dim3(p.slices);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = cmb_sm;
  if ((e = cudaLaunchKernelEx(&cfg, attend_combine_kernel, p)) != cudaSuccess)
    return cuda_fail(e, (std::string(f) + ": launch").c_str());
  return TQ_OK;
}

// Query tokens per pass of a prefill: as many as keep the virtual heads at 8 or fewer.
int prefill_qpass(int Hg) { return std::max(1, 8 / Hg); }

// One launch: the passes over the cache are work slices of their own.
PassGeom prefill_geom(int32_t Hq, int32_t Qn, int64_t T, int32_t d, int Hg) {
  const int qp = std::min(prefill_qpass(Hg), (int)Qn);
  return PassGeom{qp, (Qn + qp - 1) / qp, Qn, (int64_t)Qn * Hq * d, (int64_t)Hq * d, T - Qn + 1};
}

size_t prefill_ws(int32_t B, int32_t Hq, int32_t Hkv, int32_t Qn, int64_t T, int32_t d, int nsm) {
  const PassGeom g = prefill_geom(Hq, Qn, T, d, Hq / Hkv);
  AttPlan pl;
  att_plan(B, Hq, Hkv, T, d, nsm, pl, g.nqry, g.npass);
  return pl.total;
}
}  // namespace

// Decode attention over T tokens of every slice, whose records lie tstride apart (tstride >= T).
tq_status attend_impl(const char* f, const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                      int32_t Hkv, int64_t T, int64_t tstride, int32_t d, const void* q, int32_t q_dtype,
                      const void* rot, const uint32_t* k_codes, const uint16_t* k_norms, const uint32_t* k_signs,
                      const uint16_t* k_gammas, const uint32_t* v_codes, const uint32_t* v_signs,
                      const uint16_t* v_norms, const uint16_t* v_gammas, float scale, float* out, void* ws,
                      size_t ws_bytes, void* stream) {
  tq_status st = attend_check(f, cb_k, cb_v, B, Hq, Hkv, T, tstride, d, q, q_dtype, rot, k_codes, k_norms, k_signs,
                              k_gammas, v_codes, v_signs, v_norms, v_gammas, out, ws);
  if (st != TQ_OK) return st;
  if (ws_bytes < tq_attend_workspace_bytes(B, Hq, Hkv, T, d))
    return fail(TQ_ERR_WORKSPACE, std::string(f) + ": workspace too small");
  PassGeom g{1, 1, 1, (int64_t)Hq * d, 0, T};
  return attend_pass(f, cb_k, cb_v, B, Hq, Hkv, T, tstride, d, q, q_dtype, rot, k_codes, k_norms, k_signs, k_gammas,
                     v_codes, v_signs, v_norms, v_gammas, scale, out, ws, ws_bytes, stream, g);
}
}  // namespace tq

extern "C" TQ_API tq_status tq_attend_decode(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                             int32_t Hkv, int64_t T, int32_t d, const void* q, int32_t q_dtype,
                                             const void* rot, const uint32_t* k_codes, const uint16_t* k_norms,
                                             const uint32_t* k_signs, const uint16_t* k_gammas,
                                             const uint32_t* v_codes, const uint32_t* v_signs, const uint16_t* v_norms,
                                             const uint16_t* v_gammas, float scale, float* out, void* ws,
                                             size_t ws_bytes, void* stream) {
  clear_error();
  return attend_impl("tq_attend_decode", cb_k, cb_v, B, Hq, Hkv, T, T, d, q, q_dtype, rot, k_codes, k_norms, k_signs,
                     k_gammas, v_codes, v_signs, v_norms, v_gammas, scale, out, ws, ws_bytes, stream);
}

extern "C" TQ_API size_t tq_attend_prefill_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t Qn, int64_t T,
                                                           int32_t d) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Qn <= 0 || T < Qn || d <= 0 || Hq % Hkv) return 0;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      nsm <= 0) {
    cudaGetLastError();
    nsm = 148;
  }
  return prefill_ws(B, Hq, Hkv, Qn, T, d, nsm);
}

extern "C" TQ_API tq_status tq_attend_prefill(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                              int32_t Hkv, int32_t Qn, int64_t T, int32_t d, const void* q,
                                              int32_t q_dtype, const void* rot, const uint32_t* k_codes,
                                              const uint16_t* k_norms, const uint32_t* k_signs,
                                              const uint16_t* k_gammas, const uint32_t* v_codes,
                                              const uint32_t* v_signs, const uint16_t* v_norms,
                                              const uint16_t* v_gammas, float scale, float* out, void* ws,
                                              size_t ws_bytes, void* stream) {
  clear_error();
  const char* f = "tq_attend_prefill";
  if (Qn <= 0 || T < Qn) return fail(TQ_ERR_INVALID_ARG, "tq_attend_prefill: need 1 <= Qn <= T");
  tq_status st = attend_check(f, cb_k, cb_v, B, Hq, Hkv, T, T, d, q, q_dtype, rot, k_codes, k_norms, k_signs, k_gammas,
                              v_codes, v_signs, v_norms, v_gammas, out, ws);
  if (st != TQ_OK) return st;
  if (ws_bytes < tq_attend_prefill_workspace_bytes(B, Hq, Hkv, Qn, T, d))
    return fail(TQ_ERR_WORKSPACE, "tq_attend_prefill: workspace too small");
  // query token j (0-based among the Qn new tokens) sits at cache position T - Qn + j and sees the
  // tokens t <= T - Qn + j; every pass reads all T slots (a pass's last few chunks are masked)
  const PassGeom g = prefill_geom(Hq, Qn, T, d, Hq / Hkv);
  return attend_pass(f, cb_k, cb_v, B, Hq, Hkv, T, T, d, q, q_dtype, rot, k_codes, k_norms, k_signs, k_gammas, v_codes,
                     v_signs, v_norms, v_gammas, scale, out, ws, ws_bytes, stream, g);
}

extern "C" TQ_API size_t tq_attend_append_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t T_cur, int32_t d,
                                                          int32_t k_bits, int32_t v_codebook_bits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T_cur < 0 || d <= 0 || d % 32 || Hq % Hkv || k_bits < 1 || k_bits > 4 ||
      v_codebook_bits < 1 || v_codebook_bits > 4)
    return 0;
  return tq_attend_workspace_bytes(B, Hq, Hkv, T_cur + 1, d);
}

// tq_attend_append: one decode step on a packed KV cache with room to grow. The prep kernel encodes
// each slice's new key (Algorithm 1) and value (Algorithm 2) into slot T_cur (ai-navigate-news page:
// keys by Algorithm 1, values by Algorithm 2, appended as tokens are generated), then the main and
// combine kernels attend over the T_cur + 1 filled slots: three launches in all.
extern "C" TQ_API tq_status tq_attend_append(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                             int32_t Hkv, int64_t T_cur, int64_t T_max, int32_t d, const void* q,
                                             int32_t q_dtype, const void* k_new, const void* v_new, int32_t x_dtype,
                                             const void* rot, uint32_t* k_codes, uint16_t* k_norms,
                                             uint32_t* v_codes, uint32_t* v_signs, uint16_t* v_norms,
                                             uint16_t* v_gammas, float scale, float* out, void* ws, size_t ws_bytes,
                                             void* stream) {
  clear_error();
  const char* f = "tq_attend_append";
  if (!k_new || !v_new || !v_signs || !v_gammas)
    return fail(TQ_ERR_INVALID_ARG, "tq_attend_append: NULL pointer (values are Algorithm 2: signs and gammas are required)");
  if (T_cur < 0 || T_max < T_cur + 1) return fail(TQ_ERR_INVALID_ARG, "tq_attend_append: need 0 <= T_cur < T_max");
  if (x_dtype != TQ_F32 && x_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, "tq_attend_append: k_new / v_new dtype");
  const int64_t T = T_cur + 1;
  tq_status st = attend_check(f, cb_k, cb_v, B, Hq, Hkv, T, T_max, d, q, q_dtype, rot, k_codes, k_norms, nullptr,
                              nullptr, v_codes, v_signs, v_norms, v_gammas, out, ws);
  if (st != TQ_OK) return st;
  if (ws_bytes < tq_attend_workspace_bytes(B, Hq, Hkv, T, d))
    return fail(TQ_ERR_WORKSPACE, "tq_attend_append: workspace too small");
  const AppendArgs app{k_new, v_new, x_dtype, T_cur, k_codes, k_norms, v_codes, v_signs, v_norms, v_gammas};
  PassGeom g{1, 1, 1, (int64_t)Hq * d, 0, T};
  return attend_pass(f, cb_k, cb_v, B, Hq, Hkv, T, T_max, d, q, q_dtype, rot, k_codes, k_norms, nullptr, nullptr,
                     v_codes, v_signs, v_norms, v_gammas, scale, out, ws, ws_bytes, stream, g, &app);
}
