// Inner-product scores of queries against packed database vectors, and the top-k per query
// (tq_scores).
//
// Method (aiboss88 page: inner-product mode with unbiased estimates; vector-database nearest
// neighbour search): <q, x_hat> = n (<q', c[idx]> + alpha gamma <q'', 2z - 1>), q' = Pi q,
// q'' = S q, evaluated from the codes. With the Walsh expansion of the symmetric codebook,
// c[idx] = sum_S beta_S prod_{p in S}(1 - 2 bit_p) (odd subsets S of the bit planes, b_S = XOR of
// the planes in S):
//   <q', c[idx]> = Q sum_S beta_S - 2 sum_S beta_S <q', b_S>,      Q = sum_i q'_i.
// So one GEMM over K = (Walsh planes + sign plane) x d gives every (vector, query) pair:
//   A[v][(S, i)] = b_S,v,i (fp16 0 / 1, exact);  A[v][(sign, i)] = gamma_v (2 z_v,i - 1) (fp16, exact),
//   B[q][(S, i)] = -2 beta_S q'_i;               B[q][(sign, i)] = alpha q''_i,
// with B split into two fp16 parts (hi + 2^-11 lo, about 22 bits) that occupy two MMA columns.
// score = n_v (Q_q sum beta + D_hi + 2^-11 D_lo), scaled back by the query's power of two.
//
// Kernels: rotate (q', q'' in fp64, per-query constants), image (B operand as shared-memory
// images in global memory), main (persistent tcgen05 f16 GEMM: the A operand is expanded from the
// packed codes on the fly, 128 vectors x 128 queries per work item, scores written row-major),
// topk (per query: k largest of a chunk of scores merged into the running list). When only the
// top-k is wanted the database is processed in chunks so the score buffer stays bounded.
//
// Main-kernel roles (10 warps): 0 bulk-copies B blocks; 1 owns TMEM and issues the MMAs; 2-5 expand
// the codes of the M-tile (thread = vector) into the A ring; 6-9 epilogue (thread = vector).
// All waits are bounded (sm100.cuh).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <string>

#include "sm100.cuh"
#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kScThreads = 320;
constexpr int kMaxPlanes = 9;          // 8 Walsh planes (4-bit codes) + the sign plane
constexpr int kARing = 4, kBRing = 3;
constexpr int kQT = 128;               // queries per N-tile (256 MMA columns: hi, lo)
constexpr int kNCH = 32768;            // database vectors per chunk when only the top-k is wanted
constexpr int kMaxK = 16;
constexpr uint32_t kABytes = 128 * 128;       // one A block: 128 vectors x 64 fp16
constexpr uint32_t kBBytes = 256 * 128;       // one B block: 256 rows x 64 fp16

struct ScParams {
  int64_t n;                 // vectors in this launch
  int d, G, bc, mk, npl, vs; // code bits, Walsh planes, planes in all, sign plane?
  int nq, ntq, mtiles, nkb;  // queries, query tiles, vector tiles, 64-coordinate blocks
  int wmask[8];
  float beta[8];
  float alpha, bmax;
  const void* q;
  int q_bf16;
  const float* Pi;
  const float* S;
  const uint32_t* codes;
  const uint32_t* signs;
  const uint16_t* norms;
  const uint16_t* gammas;
  double* qp;                // [nq][d]  q' = Pi q
  double* qpp;               // [nq][d]  q'' = S q
  double* qF;                // [nq]     2^F (B scale)
  float* qc;                 // [nq]     Q sum(beta)
  float* qs;                 // [nq]     2^-F (B scale)
  uint8_t* bimg;             // [ntq][nkb * npl][kBBytes]
  float* out;                // scores, row q at out + q * ld
  int64_t ld;
  uint32_t* err;
};

// ------------------------------------------------------------------------------------------------
// rotate: q' = Pi q, q'' = S q (fp64), Q sum(beta), the power-of-two scale of the B operand
// ------------------------------------------------------------------------------------------------
__global__ void scores_rotate_kernel(const __grid_constant__ ScParams p) {
  extern __shared__ double sq[];                 // [d]
  __shared__ double red[2][8];
  const int qi = blockIdx.x, d = p.d, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int j = tid; j < d; j += blockDim.x)
    sq[j] = p.q_bf16 ? (double)__uint_as_float((uint32_t)((const uint16_t*)p.q)[(size_t)qi * d + j] << 16)
                     : (double)((const float*)p.q)[(size_t)qi * d + j];
  __syncthreads();
  double qsum = 0.0, m1 = 0.0, m2 = 0.0;
  for (int r = warp; r < d; r += blockDim.x / 32) {
    const float* prow = p.Pi + (size_t)r * d;
    const float* srow = p.S + (size_t)r * d;
    double a = 0.0, b = 0.0;
    for (int j = lane; j < d; j += 32) {
      a = fma((double)prow[j], sq[j], a);
      if (p.vs) b = fma((double)srow[j], sq[j], b);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    if (lane == 0) {
      p.qp[(size_t)qi * d + r] = a;
      p.qpp[(size_t)qi * d + r] = b;
      qsum += a;
      m1 = fmax(m1, fabs(a));
      m2 = fmax(m2, fabs(b));
    }
  }
  if (lane == 0) {
    red[0][warp] = qsum;
    red[1][warp] = fmax(2.0 * p.bmax * m1, (double)p.alpha * m2);
  }
  __syncthreads();
  if (tid == 0) {
    double Q = 0.0, vmax = 0.0;
    for (int w = 0; w < (int)blockDim.x / 32; ++w) {
      Q += red[0][w];
      vmax = fmax(vmax, red[1][w]);
    }
    double sb = 0.0;
    for (int s = 0; s < p.mk; ++s) sb += (double)p.beta[s];
    int F = 0;
    if (vmax > 0.0) {
      int E;
      frexp(vmax, &E);               // vmax < 2^E
      F = 14 - E;                    // |B| * 2^F < 2^14
    }
    p.qc[qi] = (float)(Q * sb);
    p.qs[qi] = (float)ldexp(1.0, -F);
    p.qF[qi] = ldexp(1.0, F);
  }
}

// element e (0..63) of a 64-coordinate block -> coordinate offset inside the block: output word
// j = e / 2 of the expansion holds bits (j % 16) and (j % 16) + 16 of plane word j / 16
__host__ __device__ inline int elem_coord(int e) {
  const int j = e >> 1, h = e & 1;
  return 32 * (j >> 4) + (j & 15) + 16 * h;
}

// ------------------------------------------------------------------------------------------------
// image: the B operand, per (query tile, block (kb, plane)) one K-major SW128 image of 256 rows
// (query q -> rows 2q (hi) and 2q+1 (lo)) x 64 fp16
// ------------------------------------------------------------------------------------------------
__global__ void scores_image_kernel(const __grid_constant__ ScParams p) {
  const int64_t total = (int64_t)p.ntq * kQT * p.npl * p.d;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int d = p.d;
  const int e = (int)(idx % 64);
  int64_t rest = idx / 64;
  const int S = (int)(rest % p.npl);
  rest /= p.npl;
  const int kb = (int)(rest % p.nkb);
  const int qg = (int)(rest / p.nkb);            // global query index (may be a pad)
  const int nt = qg / kQT, ql = qg % kQT;
  const int coord = kb * 64 + elem_coord(e);
  float hi = 0.0f, lo = 0.0f;
  if (qg < p.nq) {
    const double scale = p.qF[qg];
    const double v = (S < p.mk ? -2.0 * (double)p.beta[S] * p.qp[(size_t)qg * d + coord]
                               : (double)p.alpha * p.qpp[(size_t)qg * d + coord]) * scale;
    const __half h = __double2half(v);
    hi = __half2float(h);
    lo = (float)((v - (double)hi) * 2048.0);
  }
  uint8_t* blk = p.bimg + ((size_t)nt * p.nkb * p.npl + (size_t)kb * p.npl + S) * kBBytes;
  *(__half*)(blk + sw128_offset(2 * ql, 2 * e, 256)) = __float2half_rn(hi);
  *(__half*)(blk + sw128_offset(2 * ql + 1, 2 * e, 256)) = __float2half_rn(lo);
}

// ------------------------------------------------------------------------------------------------
// main: tcgen05 f16 GEMM with the A operand expanded from the codes
// ------------------------------------------------------------------------------------------------
enum ScBars {
  A_FULL = 0,                  // [kARing] expanders -> MMA (4 warps)
  A_EMPTY = A_FULL + kARing,   // [kARing] MMA commit
  B_FULL = A_EMPTY + kARing,   // [kBRing] bulk copy
  B_EMPTY = B_FULL + kBRing,   // [kBRing] MMA commit
  ACC_FULL = B_EMPTY + kBRing, // [2] MMA commit
  ACC_EMPTY = ACC_FULL + 2,    // [2] epilogue (4 warps)
  SC_NBARS = ACC_EMPTY + 2
};

struct ScLayout {
  uint32_t off_a, off_b, off_bar, total;
};
__host__ __device__ inline ScLayout sc_layout() {
  ScLayout L{};
  L.off_a = 0;
  L.off_b = kARing * kABytes;
  L.off_bar = L.off_b + kBRing * kBBytes;
  L.total = L.off_bar + 64 * 8 + 1024;
  return L;
}

__global__ void __launch_bounds__(kScThreads, 1) scores_main_kernel(const __grid_constant__ ScParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const ScLayout Lo = sc_layout();
  uint64_t* bar = (uint64_t*)(smem + Lo.off_bar);
  uint32_t* tmem_slot = (uint32_t*)(bar + SC_NBARS);
  volatile uint32_t* abort_flag = (volatile uint32_t*)(bar + SC_NBARS) + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nitems = p.mtiles * p.ntq;
  const int nblk = p.nkb * p.npl;                 // K blocks per work item
  const int G = p.G, bc = p.bc;

  if (tid == 0) {
    for (int s = 0; s < kARing; ++s) {
      mbar_init(&bar[A_FULL + s], 4);
      mbar_init(&bar[A_EMPTY + s], 1);
    }
    for (int s = 0; s < kBRing; ++s) {
      mbar_init(&bar[B_FULL + s], 1);
      mbar_init(&bar[B_EMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[ACC_FULL + s], 1);
      mbar_init(&bar[ACC_EMPTY + s], 4);
    }
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

  if (warp == 0) {
    // ------------------------------------ producer: B blocks ---------------------------------------
    // warp-uniform schedule; one elected lane issues the copies
    int64_t j = 0;                                 // running block counter of this CTA
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int nt = it % p.ntq;
      const uint8_t* src = p.bimg + (size_t)nt * nblk * kBBytes;
      for (int k = 0; k < nblk; ++k, ++j) {
        const int slot = (int)(j % kBRing);
        const uint32_t use = (uint32_t)(j / kBRing);
        if (!mbar_wait_warp(&bar[B_EMPTY + slot], (use & 1) ^ 1, p.err, kDevTimeoutSync, abort_flag)) {
          ok = false;
          break;
        }
        if (elect_one_sync()) {
          mbar_arrive_expect_tx(&bar[B_FULL + slot], kBBytes);
          bulk_g2s(smem + Lo.off_b + slot * kBBytes, src + (size_t)k * kBBytes, kBBytes, &bar[B_FULL + slot]);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------ MMA issuer -----------------------------------------------
    // warp-uniform schedule (descriptors stay in uniform registers); one elected lane issues
    const uint32_t idesc = idesc_f16_f32(128, 256);
    const uint64_t da0 = desc_kmajor_sw128(smem_u32(smem + Lo.off_a));
    const uint64_t db0 = desc_kmajor_sw128(smem_u32(smem + Lo.off_b));
    int64_t j = 0;
    int li = 0;                                    // local work-item counter
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
      const int acc = li & 1;
      if (li >= 2 && !mbar_wait_warp(&bar[ACC_EMPTY + acc], ((li >> 1) - 1) & 1, p.err, kDevTimeoutSync, abort_flag))
        break;
      tc_fence_after();
      const uint32_t dcol = tbase + acc * 256;
      for (int k = 0; k < nblk; ++k, ++j) {
        const int as = (int)(j % kARing), bs = (int)(j % kBRing);
        if (!mbar_wait_warp(&bar[A_FULL + as], (uint32_t)(j / kARing) & 1, p.err, kDevTimeoutSync, abort_flag) ||
            !mbar_wait_warp(&bar[B_FULL + bs], (uint32_t)(j / kBRing) & 1, p.err, kDevTimeoutLoad, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = da0 + ((as * kABytes) >> 4);
        const uint64_t db = db0 + ((bs * kBBytes) >> 4);
        if (elect_one_sync()) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) mma_f16_ss(dcol, da + ks * 2, db + ks * 2, idesc, (k > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bar[A_EMPTY + as]);
          mma_commit(&bar[B_EMPTY + bs]);
        }
        __syncwarp();
      }
      if (ok && elect_one_sync()) mma_commit(&bar[ACC_FULL + acc]);
      __syncwarp();
    }
  } else if (warp < 6) {
    // ------------------------------------ expanders (thread = vector) ------------------------------
    const int r = (warp & 3) * 32 + lane;          // row of the M-tile (TMEM lane quarter irrelevant here)
    uint32_t soff[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) soff[ch] = sw128_offset(r, ch * 16, 128);
    int64_t j = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const int mt = it / p.ntq;
      const int64_t v = (int64_t)mt * 128 + r;
      const bool live = v < p.n;
      const uint32_t* cw = p.codes + (live ? v : 0) * G * bc;
      const uint32_t* sw = p.vs ? p.signs + (live ? v : 0) * G : nullptr;
      uint32_t gg = 0;
      if (p.vs && live) {
        const uint32_t g16 = __ldg(p.gammas + v);
        gg = g16 | (g16 << 16);
      }
      for (int kb = 0; kb < p.nkb && ok; ++kb) {
        // raw plane words of the two 32-coordinate groups of this block
        uint32_t raw[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
        uint32_t sg[2] = {0, 0};
        if (live) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int pl = 0; pl < 4; ++pl)
              if (pl < bc) raw[h][pl] = __ldg(cw + (2 * kb + h) * bc + pl);
            if (p.vs) sg[h] = __ldg(sw + 2 * kb + h);
          }
        }
        for (int S = 0; S < p.npl; ++S, ++j) {
          const int as = (int)(j % kARing);
          if (j >= kARing && !mbar_wait_warp(&bar[A_EMPTY + as], ((uint32_t)(j / kARing) - 1) & 1, p.err,
                                             kDevTimeoutMma, abort_flag)) {
            ok = false;
            break;
          }
          const bool sign_plane = p.vs && S == p.npl - 1;
          uint32_t w[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (sign_plane) {
              w[h] = sg[h];
            } else {
              const int m = p.wmask[S];
              uint32_t x = 0;
#pragma unroll
              for (int pl = 0; pl < 4; ++pl)
                if (m & (1 << pl)) x ^= raw[h][pl];
              w[h] = x;
            }
          }
          uint8_t* ab = smem + Lo.off_a + as * kABytes;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint32_t o[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int jw = ch * 4 + u;                   // output word: coordinates (jw%16, jw%16+16) of word jw/16
              const uint32_t t = w[jw >> 4] >> (jw & 15);
              o[u] = sign_plane ? (gg ^ (~(t << 15) & 0x80008000u)) : ((t & 0x00010001u) * 0x3C00u);
            }
            *(uint4*)(ab + soff[ch]) = make_uint4(o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[A_FULL + as]);
        }
      }
    }
  } else {
    // ------------------------------------ epilogue (thread = vector) -------------------------------
    const int qw = warp & 3;                        // TMEM lane quarter of this warp
    const int r = qw * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qw * 32) << 16;
    int li = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
      const int acc = li & 1;
      const int mt = it / p.ntq, nt = it % p.ntq;
      if (!mbar_wait_warp(&bar[ACC_FULL + acc], (li >> 1) & 1, p.err, kDevTimeoutMma, abort_flag)) break;
      tc_fence_after();
      const int64_t v = (int64_t)mt * 128 + r;
      const bool live = v < p.n;
      const float nv = live ? __half2float(__ushort_as_half(__ldg(p.norms + v))) : 0.0f;
      for (int c16 = 0; c16 < 16; ++c16) {
        uint32_t x[16];
        tmem_ld16(tbase + lane_base + acc * 256 + c16 * 16, x);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int qg = nt * kQT + c16 * 8 + u;
          if (live && qg < p.nq) {
            const float dv = fmaf(__uint_as_float(x[2 * u + 1]), 1.0f / 2048.0f, __uint_as_float(x[2 * u]));
            p.out[(size_t)qg * p.ld + v] = nv * fmaf(dv, __ldg(p.qs + qg), __ldg(p.qc + qg));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[ACC_EMPTY + acc]);
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
// top-k: per query, the k largest scores (ties to the lower id) of a row of `cnt` scores whose
// ids start at id0, merged with the running list already in ids/vals when `merge` is set
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ bool better(float a, int64_t ia, float b, int64_t ib) {
  return a > b || (a == b && ia < ib);
}

__global__ void __launch_bounds__(256) scores_topk_kernel(const float* __restrict__ sc, int64_t ld, int64_t cnt,
                                                          int64_t id0, int k, int merge, int32_t* ids, float* vals) {
  const int qi = blockIdx.x, tid = threadIdx.x;
  const float* row = sc + (size_t)qi * ld;
  float lv[kMaxK];
  int64_t li[kMaxK];
  int nl = 0;
#pragma unroll
  for (int i = 0; i < kMaxK; ++i) {
    lv[i] = -INFINITY;
    li[i] = INT64_MAX;
  }
  auto insert = [&](float s, int64_t id) {
    // lv / li stay sorted best first; a candidate enters if the list is short or it beats the last
    if (nl == k && !better(s, id, lv[k - 1], li[k - 1])) return;
    int i = nl < k ? nl : k - 1;
    while (i > 0 && better(s, id, lv[i - 1], li[i - 1])) {
      lv[i] = lv[i - 1];
      li[i] = li[i - 1];
      --i;
    }
    lv[i] = s;
    li[i] = id;
    if (nl < k) ++nl;
  };
  for (int64_t c = tid; c < cnt; c += blockDim.x) insert(row[c], id0 + c);
  if (merge && tid < k) {
    const int32_t pid = ids[(size_t)qi * k + tid];
    if (pid >= 0) insert(vals[(size_t)qi * k + tid], pid);
  }
  // block merge: k rounds of a block-wide argmax over the heads of the sorted local lists
  __shared__ float bv[8];
  __shared__ long long bi[8];
  __shared__ int bt[8];
  __shared__ long long wi;
  __shared__ int wt;
  int head = 0;
  for (int round = 0; round < k; ++round) {
    const float v0 = head < nl ? lv[head] : -INFINITY;
    const int64_t id0h = head < nl ? li[head] : INT64_MAX;
    float v = v0;
    int64_t id = id0h;
    int owner = tid;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, o);
      const long long oi = __shfl_xor_sync(0xffffffffu, (long long)id, o);
      const int ot = __shfl_xor_sync(0xffffffffu, owner, o);
      if (better(ov, oi, v, id)) {
        v = ov;
        id = oi;
        owner = ot;
      }
    }
    if ((tid & 31) == 0) {
      bv[tid >> 5] = v;
      bi[tid >> 5] = id;
      bt[tid >> 5] = owner;
    }
    __syncthreads();
    if (tid == 0) {
      float b = bv[0];
      long long i0 = bi[0];
      int t0 = bt[0];
      for (int w = 1; w < (int)blockDim.x / 32; ++w)
        if (better(bv[w], bi[w], b, i0)) {
          b = bv[w];
          i0 = bi[w];
          t0 = bt[w];
        }
      wi = i0;
      wt = t0;
      const bool valid = i0 != INT64_MAX;
      ids[(size_t)qi * k + round] = valid ? (int32_t)i0 : -1;
      vals[(size_t)qi * k + round] = valid ? b : -INFINITY;
    }
    __syncthreads();
    if (tid == wt && wi != INT64_MAX) ++head;
    __syncthreads();
  }
}

}  // namespace
}  // namespace tq

using namespace tq;

namespace {

struct ScPlan {
  int ntq, nkb;
  size_t off_qp, off_qpp, off_qF, off_qc, off_qs, off_img, off_chunk, total;
};

ScPlan sc_plan(int64_t nq, int64_t n, int d, int k) {
  ScPlan P{};
  auto al = [](size_t x) { return (x + 1023) / 1024 * 1024; };
  P.ntq = (int)((nq + kQT - 1) / kQT);
  P.nkb = d / 64;
  size_t off = 0;
  P.off_qp = off; off += al((size_t)nq * d * sizeof(double));
  P.off_qpp = off; off += al((size_t)nq * d * sizeof(double));
  P.off_qF = off; off += al((size_t)nq * sizeof(double));
  P.off_qc = off; off += al((size_t)nq * sizeof(float));
  P.off_qs = off; off += al((size_t)nq * sizeof(float));
  P.off_img = off; off += al((size_t)P.ntq * P.nkb * kMaxPlanes * kBBytes);
  P.off_chunk = off;
  if (k > 0) off += al((size_t)nq * std::min<int64_t>(std::max<int64_t>(n, 1), kNCH) * sizeof(float));
  P.total = off;
  return P;
}

}  // namespace

extern "C" TQ_API size_t tq_scores_workspace_bytes(int64_t nq, int64_t n, int32_t d, int32_t k) {
  if (nq <= 0 || n < 0 || d <= 0 || d % 64 || k < 0) return 0;
  return sc_plan(nq, n, d, k).total;
}

extern "C" TQ_API tq_status tq_scores(const tq_codebook* cb, int64_t nq, int64_t n, int32_t d, const void* q,
                                      int32_t q_dtype, const void* rot, const uint32_t* codes, const uint32_t* signs,
                                      const uint16_t* norms, const uint16_t* gammas, float* scores, int32_t k,
                                      int32_t* topk_ids, float* topk_scores, void* ws, size_t ws_bytes,
                                      void* stream) {
  clear_error();
  const std::string f = "tq_scores";
  if (!cb || !q || !rot || !ws) return fail(TQ_ERR_INVALID_ARG, f + ": NULL pointer");
  if (n > 0 && (!codes || !norms)) return fail(TQ_ERR_INVALID_ARG, f + ": NULL codes or norms");
  if ((signs == nullptr) != (gammas == nullptr))
    return fail(TQ_ERR_INVALID_ARG, f + ": signs and gammas must both be NULL or both be set");
  if (nq <= 0 || n < 0 || k < 0) return fail(TQ_ERR_INVALID_ARG, f + ": bad nq / n / k");
  if (d <= 0 || d % 64 || d > 4096) return fail(TQ_ERR_UNSUPPORTED, f + ": d must be a multiple of 64 up to 4096");
  if (k > kMaxK) return fail(TQ_ERR_UNSUPPORTED, f + ": k must be at most 16");
  if (k > 0 && (!topk_ids || !topk_scores)) return fail(TQ_ERR_INVALID_ARG, f + ": k > 0 needs topk_ids and topk_scores");
  if (k == 0 && !scores) return fail(TQ_ERR_INVALID_ARG, f + ": nothing to compute (scores NULL and k = 0)");
  if (n > INT32_MAX) return fail(TQ_ERR_UNSUPPORTED, f + ": ids are int32");
  if (cb->d != d) return fail(TQ_ERR_INVALID_ARG, f + ": codebook d mismatch");
  if (cb->bits < 1 || cb->bits > 4 || cb->levels != (1 << cb->bits)) return fail(TQ_ERR_INVALID_ARG, f + ": bad codebook");
  for (int i = 0; i < cb->levels; ++i)
    if (cb->c[cb->levels - 1 - i] != -cb->c[i]) return fail(TQ_ERR_INVALID_ARG, f + ": codebook not symmetric");
  if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return fail(TQ_ERR_UNSUPPORTED, f + ": q dtype");
  if (!aligned16(ws) || !aligned16(rot) || (codes && !aligned16(codes)) || (signs && !aligned16(signs)))
    return fail(TQ_ERR_INVALID_ARG, f + ": pointers must be 16-byte aligned");
  const ScPlan P = sc_plan(nq, n, d, k);
  if (ws_bytes < P.total) return fail(TQ_ERR_WORKSPACE, f + ": workspace too small");

  ScParams p{};
  p.d = d;
  p.G = d / 32;
  p.bc = cb->bits;
  p.mk = walsh_planes(cb, p.wmask, p.beta);
  p.vs = signs ? 1 : 0;
  p.npl = p.mk + p.vs;
  p.nq = (int)nq;
  p.ntq = P.ntq;
  p.nkb = P.nkb;
  p.alpha = (float)(std::sqrt(M_PI / 2.0) / d);
  p.bmax = 0.0f;
  for (int i = 0; i < p.mk; ++i) p.bmax = std::max(p.bmax, std::fabs(p.beta[i]));
  p.q = q;
  p.q_bf16 = q_dtype == TQ_BF16;
  const RotLayout RL = rot_layout(d);
  p.Pi = (const float*)((const char*)rot + RL.pi32);
  p.S = (const float*)((const char*)rot + RL.s32);
  p.norms = norms;
  p.gammas = gammas;
  uint8_t* w = (uint8_t*)ws;
  p.qp = (double*)(w + P.off_qp);
  p.qpp = (double*)(w + P.off_qpp);
  p.qF = (double*)(w + P.off_qF);
  p.qc = (float*)(w + P.off_qc);
  p.qs = (float*)(w + P.off_qs);
  p.bimg = w + P.off_img;
  p.err = device_error_word();
  if (!p.err) return fail(TQ_ERR_CUDA, f + ": no device error word");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;

  scores_rotate_kernel<<<(int)nq, 256, (size_t)d * sizeof(double), st>>>(p);
  {
    const int64_t tot = (int64_t)P.ntq * kQT * p.npl * d;
    scores_image_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(p);
  }
  const ScLayout Lo = sc_layout();
  e = cudaFuncSetAttribute(scores_main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lo.total);
  if (e != cudaSuccess) return cuda_fail(e, "tq_scores: shared memory attribute");
  const int nsm = sm_count();
  auto run_main = [&](int64_t v0, int64_t cnt, float* out, int64_t ld) {
    ScParams c = p;
    c.n = cnt;
    c.codes = codes + v0 * p.G * p.bc;
    c.signs = signs ? signs + v0 * p.G : nullptr;
    c.norms = norms + v0;
    c.gammas = gammas ? gammas + v0 : nullptr;
    c.mtiles = (int)((cnt + 127) / 128);
    c.out = out;
    c.ld = ld;
    const int items = c.mtiles * c.ntq;
    scores_main_kernel<<<std::min(items, nsm), kScThreads, Lo.total, st>>>(c);
  };
  if (n == 0) {
    if (k > 0) {
      scores_topk_kernel<<<(int)nq, 256, 0, st>>>(nullptr, 0, 0, 0, k, 0, topk_ids, topk_scores);
    }
  } else if (scores) {
    run_main(0, n, scores, n);
    if (k > 0) scores_topk_kernel<<<(int)nq, 256, 0, st>>>(scores, n, n, 0, k, 0, topk_ids, topk_scores);
  } else {
    float* chunk = (float*)(w + P.off_chunk);
    const int64_t nch = std::min<int64_t>(n, kNCH);
    for (int64_t v0 = 0; v0 < n; v0 += nch) {
      const int64_t cnt = std::min<int64_t>(nch, n - v0);
      run_main(v0, cnt, chunk, nch);
      scores_topk_kernel<<<(int)nq, 256, 0, st>>>(chunk, nch, cnt, v0, k, v0 > 0 ? 1 : 0, topk_ids, topk_scores);
    }
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "tq_scores: launch");
  return TQ_OK;
}
