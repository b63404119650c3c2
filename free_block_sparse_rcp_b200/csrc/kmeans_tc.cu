// Lloyd k-means of the response-coupled partition (gist.science technical summary,
// section 2.A), scored in the raw d-dimensional space on the tensor cores.
//
// Keys are clustered on y = A k with A = Lambda_r^{1/2} U_r^T (r_e x d), queries on
// z = A q with A = s C (G_k x d).  A centroid in coordinate space is nu_g = A m_g where
// m_g is the mean raw row of the cluster (a mean commutes with the linear map), so
//   ||y - nu_g||^2 = ||y||^2 + ||nu_g||^2 - 2 x . w_g,     w_g = A^T nu_g  (d-vector).
// The assignment therefore needs only the bf16 input rows x (exact) against the weights
// w_g (split into bf16 hi + lo) on the tensor cores: score_g = ||nu_g||^2 - 2 x.w_g.
// The argmin is accepted when the runner-up's score is further away than twice a
// rigorous error bound of the split-bf16 products and fp32 accumulation; otherwise the
// row is re-assigned by the exact fp32 direct form sum_c (y_c - nu_gc)^2 (ties -> lowest
// g), which is the semantics the coordinates-based definition has.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace spr {
namespace km {

using namespace spr::tc;

// ---------------------------------------------------------------------------
// Seeds: m_g = x_{init_g} (fp32), init_g = g-th row of the stream's draw.
// grid = BH, block = 256.
// ---------------------------------------------------------------------------
constexpr int kMapCap = 4096;

__global__ void __launch_bounds__(256) k_seed_rows(const __nv_bfloat16* __restrict__ X, int N, int d, int G,
                                                  uint64_t seed, HeadMap hm, int purpose, float* __restrict__ m,
                                                  int* __restrict__ init_out, int* err) {
  extern __shared__ __align__(16) unsigned char smem_seed[];
  int* sidx = reinterpret_cast<int*>(smem_seed);   // [G] drawn rows
  int* jbuf = sidx + G;                             // [G] the draws' offsets
  const int bh = blockIdx.x, tid = threadIdx.x;
  if (!draw_without_replacement_block(stream_state(seed, hm.global(bh), purpose), N, G, kMapCap, sidx, jbuf)) {
    if (tid == 0) set_error(err, DERR_DRAW);
    return;
  }
  // 16-byte pieces of the drawn rows (rows are 16-byte aligned: d is a multiple of 8), four
  // loads in flight per thread
  const int VPR = d / 8;
#pragma unroll 4
  for (int e = tid; e < G * VPR; e += blockDim.x) {
    const int g = e / VPR, v = e - g * VPR;
    const uint4 x = *reinterpret_cast<const uint4*>(X + ((size_t)bh * N + sidx[g]) * d + v * 8);
    const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
    const float2 f0 = __bfloat1622float2(x2[0]), f1 = __bfloat1622float2(x2[1]);
    const float2 f2 = __bfloat1622float2(x2[2]), f3 = __bfloat1622float2(x2[3]);
    float4* dst = reinterpret_cast<float4*>(m + ((size_t)bh * G + g) * d + v * 8);
    dst[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
    dst[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
  }
  if (init_out)
    for (int g = tid; g < G; g += blockDim.x) init_out[(size_t)bh * G + g] = sidx[g];
}

// ---------------------------------------------------------------------------
// Centroid weights.  A(j, c) = a_scale * A[j * sj + c * sc] (D x d) is staged once per
// CTA in shared memory as sA[j][c] with row stride d + 1 (conflict-free both ways).
// One warp per group (16 groups per CTA).
// mode 0: m holds the centroids (the seeds).
// mode 1: m_g = (sum of the rows assigned to g) / (their count): the partial sums the
//         previous assignment pass left per segment of the head, added in segment order
//         in fp64 (the group's warp, four columns per lane, the loads of eight segments in
//         flight), then the label corrections of the exact re-check applied in ascending
//         row order (a row moves from its provisional group to its final one); an empty
//         group keeps its centroid.  m is updated in place.
// mode 2: as mode 1 but an empty group gets 0, the means are written to m and no weights
//         are formed (the K/V group centroids after the last pass).
// Weights: nu = A m (fp32, sequential over c), bias = ||nu||^2, w = A^T nu (sequential over
//   j) -> w_hi = bf16(w), w_lo = bf16(w - w_hi); wnorm = ||w||.
// Rows g in [G, GP) are padding: w = 0, bias = +inf.
// grid = (ceil(GP / WG_PER_CTA), BH), block = 512.
// ---------------------------------------------------------------------------
constexpr int WG_PER_CTA = 16;
constexpr int CW_THREADS = 512;
constexpr int kCorrCap = 2048;   // corrections of one CTA's groups per pass

// floats of the region that holds A for the weights and, before that, the segment-slot rows
// and counts of the CTA's groups and its sorted corrections
__host__ __device__ inline int cw_scratch_floats(int d, int D, int SPH) {
  const int a = D * (d + 1), b = 2 * SPH * WG_PER_CTA + 2 * kCorrCap;
  return ((a > b ? a : b) + 3) & ~3;
}

struct KmPartials {
  const unsigned char* slots; // [BH][SPH] segment slots of the assignment pass (kmeans_slot_bytes each)
  const int* corr_count;      // [BH]
  const int4* corr;           // [BH][N] (row, provisional label, final label, -)
  const __nv_bfloat16* X;     // rows
  int N, SPH;
};

__global__ void __launch_bounds__(CW_THREADS) k_centroid_weights(float* __restrict__ m, int G, int GP, int d,
                                                                const float* __restrict__ A, size_t a_head, int sj,
                                                                int sc, float a_scale, int D, int DT, int mode,
                                                                KmPartials pp, float* __restrict__ nu,
                                                                float* __restrict__ bias, float* __restrict__ wnorm,
                                                                __nv_bfloat16* __restrict__ w_hi,
                                                                __nv_bfloat16* __restrict__ w_lo, int* err) {
  extern __shared__ __align__(16) float sw[];
  double* acc = reinterpret_cast<double*>(sw);               // [WG_PER_CTA][d]
  int* cnt = reinterpret_cast<int*>(acc + WG_PER_CTA * d);   // [WG_PER_CTA]
  float* sA = reinterpret_cast<float*>(cnt + WG_PER_CTA);    // [D][d + 1]  (the means phase uses it as scratch)
  float* sMg = sA + cw_scratch_floats(d, D, pp.SPH);         // [WG_PER_CTA][d] this CTA's centroids
  float* sNu = sMg + WG_PER_CTA * d;                         // [WG_PER_CTA][128] their nu
  const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g0 = blockIdx.x * WG_PER_CTA, g1 = min(GP, g0 + WG_PER_CTA);
  static_assert(WG_PER_CTA == CW_THREADS / 32, "one group per warp");
  if (mode != 0) {
    // ---- means from the partial sums of the previous pass: the head's segment slots in
    // segment order (the mean's definition, summed in fp64); the slot of a segment holds
    // only the groups that occur in it
    const size_t sbytes = (size_t)GP * 8 + (size_t)GP * d * 4;
    const unsigned char* hs = pp.slots + (size_t)bh * pp.SPH * sbytes;
    int* spos = reinterpret_cast<int*>(sA);                   // [SPH][WG_PER_CTA] slot rows
    int* scnt = spos + pp.SPH * WG_PER_CTA;                   // [SPH][WG_PER_CTA] slot counts
    int2* sel = reinterpret_cast<int2*>(scnt + pp.SPH * WG_PER_CTA);   // [kCorrCap] corrections
    __shared__ int s_nsel, s_over;
    for (int e = tid; e < pp.SPH * WG_PER_CTA; e += CW_THREADS) {
      const int sgm = e / WG_PER_CTA, gi = e - sgm * WG_PER_CTA;
      const int* smap = reinterpret_cast<const int*>(hs + (size_t)sgm * sbytes);
      const bool in = gi < g1 - g0;
      spos[e] = in ? smap[g0 + gi] : -1;
      scnt[e] = in ? smap[GP + g0 + gi] : 0;
    }
    if (tid == 0) { s_nsel = 0; s_over = 0; }
    __syncthreads();
    {
      // warp = group; lane = four columns (d = 64: lanes 0-15)
      const int gi = warp, c4 = lane * 4;
      const bool act = c4 < d;
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      constexpr int SB = 8;
      for (int sgm0 = 0; sgm0 < pp.SPH; sgm0 += SB) {
        float4 v[SB];
        int pos[SB];
#pragma unroll
        for (int q = 0; q < SB; ++q) {
          const int sgm = sgm0 + q;
          pos[q] = sgm < pp.SPH ? spos[sgm * WG_PER_CTA + gi] : -1;
          v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (pos[q] >= 0 && act)
            v[q] = *reinterpret_cast<const float4*>(hs + (size_t)sgm * sbytes + (size_t)GP * 8 +
                                                    ((size_t)pos[q] * d + c4) * 4);
        }
#pragma unroll
        for (int q = 0; q < SB; ++q)
          if (pos[q] >= 0) {
            a0 += (double)v[q].x;
            a1 += (double)v[q].y;
            a2 += (double)v[q].z;
            a3 += (double)v[q].w;
          }
      }
      if (act) {
        acc[gi * d + c4] = a0;
        acc[gi * d + c4 + 1] = a1;
        acc[gi * d + c4 + 2] = a2;
        acc[gi * d + c4 + 3] = a3;
      }
      if (lane == 0) {
        int n = 0;
        for (int sgm = 0; sgm < pp.SPH; ++sgm) n += scnt[sgm * WG_PER_CTA + gi];
        cnt[gi] = n;
      }
    }
    // the re-check's corrections that move a row out of or into this CTA's groups
    const int nc = min(pp.corr_count[bh], pp.N);
    const int4* cl = pp.corr + (size_t)bh * pp.N;
    for (int i = tid; i < nc; i += CW_THREADS) {
      const int4 cr = cl[i];
      const bool from = cr.y >= g0 && cr.y < g1, to = cr.z >= g0 && cr.z < g1;
      if (from || to) {
        if (cr.x < 0 || cr.x >= pp.N) { set_error(err, DERR_INDEX); continue; }
        const int k = atomicAdd(&s_nsel, 1);
        if (k < kCorrCap) sel[k] = make_int2(cr.x, ((from ? cr.y - g0 : 0xFF) << 8) | (to ? cr.z - g0 : 0xFF));
        else s_over = 1;
      }
    }
    __syncthreads();
    const int ns = min(s_nsel, kCorrCap);
    if (s_over) { if (tid == 0) set_error(err, DERR_CAPACITY); }
    if (ns > 0) {
      // ascending row order (bitonic sort of the selected list, padded with rows past N)
      int p2 = 1;
      while (p2 < ns) p2 <<= 1;
      for (int i = ns + tid; i < p2; i += CW_THREADS) sel[i] = make_int2(0x7fffffff, 0xFFFF);
      __syncthreads();
      for (int kk = 2; kk <= p2; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
          for (int i = tid; i < p2; i += CW_THREADS) {
            const int l = i ^ j;
            if (l > i) {
              const int2 x = sel[i], y = sel[l];
              const bool up = (i & kk) == 0;
              if ((x.x > y.x) == up) { sel[i] = y; sel[l] = x; }
            }
          }
          __syncthreads();
        }
      }
      // apply them in that order: thread c owns column c of the CTA's groups
      for (int c = tid; c < d; c += CW_THREADS) {
        for (int k = 0; k < ns; ++k) {
          const int2 e = sel[k];
          const int fi = (e.y >> 8) & 0xFF, ti = e.y & 0xFF;
          const double x = (double)bf2f(pp.X[((size_t)bh * pp.N + e.x) * d + c]);
          if (fi != 0xFF) acc[fi * d + c] -= x;
          if (ti != 0xFF) acc[ti * d + c] += x;
          if (c == 0) {
            if (fi != 0xFF) cnt[fi] -= 1;
            if (ti != 0xFF) cnt[ti] += 1;
          }
        }
      }
    }
    __syncthreads();
    for (int e = tid; e < (g1 - g0) * d; e += CW_THREADS) {
      const int gi = e / d, c = e - gi * d, g = g0 + gi;
      if (g >= G) continue;
      const int n = cnt[gi];
      if (n > 0) m[((size_t)bh * G + g) * d + c] = (float)(acc[e] / (double)n);
      else if (mode == 2) m[((size_t)bh * G + g) * d + c] = 0.f;
    }
    __syncthreads();
    if (mode == 2) return;
  }
  const float* Ah = A + a_head * bh;
  // staging loops unrolled so that each thread keeps several loads in flight; consecutive
  // threads read consecutive addresses of A (its unit-stride index runs fastest)
  if (sj == 1) {
#pragma unroll 8
    for (int e = tid; e < D * d; e += CW_THREADS) {
      const int c = e / D, j = e - c * D;
      sA[j * (d + 1) + c] = Ah[(size_t)j + (size_t)c * sc];
    }
  } else {
#pragma unroll 8
    for (int e = tid; e < D * d; e += CW_THREADS) {
      const int j = e / d, c = e - j * d;
      sA[j * (d + 1) + c] = Ah[(size_t)j * sj + (size_t)c * sc];
    }
  }
  __syncthreads();
#pragma unroll 8
  for (int e = tid; e < WG_PER_CTA * d; e += CW_THREADS) {
    const int gi = e / d, c = e - gi * d, g = g0 + gi;
    sMg[e] = (g < g1 && g < G) ? m[((size_t)bh * G + g) * d + c] : 0.f;
  }
  __syncthreads();
  // warp w forms the weights of group g0 + w; lanes split j for nu = A m and c for
  // w = A^T nu, each sum in ascending order of its index
  const int g = g0 + warp;
  const bool live = g < g1 && g < G;
  if (g < g1 && g >= G) {
    // padding group: never the argmin
    const size_t wrow = ((size_t)bh * GP + g) * d;
    for (int c = lane; c < d; c += 32) {
      w_hi[wrow + c] = __float2bfloat16(0.f);
      w_lo[wrow + c] = __float2bfloat16(0.f);
    }
    if (lane == 0) {
      bias[(size_t)bh * GP + g] = __int_as_float(0x7f800000);
      wnorm[(size_t)bh * GP + g] = 0.f;
    }
  }
  if (!live) return;
  float acc4[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const float* m0 = sMg + warp * d;
    for (int c = 0; c < d; ++c) {
      const float x0 = m0[c];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = lane + 32 * k;
        if (j < D) acc4[k] = fmaf(sA[j * (d + 1) + c], x0, acc4[k]);
      }
    }
  }
  {
    float b2 = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = lane + 32 * k;
      if (j < D) {
        const float a = acc4[k] * a_scale;
        sNu[warp * 128 + j] = a;
        b2 = fmaf(a, a, b2);
      }
    }
    b2 = warp_sum(b2);
    for (int j = lane; j < DT; j += 32) nu[((size_t)bh * G + g) * DT + j] = j < D ? sNu[warp * 128 + j] : 0.f;
    if (lane == 0) bias[(size_t)bh * GP + g] = b2;
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) acc4[k] = 0.f;
  {
    const float* n0 = sNu + warp * 128;
    for (int j = 0; j < D; ++j) {
      const float y0 = n0[j];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        if (c < d) acc4[k] = fmaf(sA[j * (d + 1) + c], y0, acc4[k]);
      }
    }
  }
  const size_t wrow = ((size_t)bh * GP + g) * d;
  float n2 = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = lane + 32 * k;
    if (c < d) {
      const float w = a_scale * acc4[k];
      n2 = fmaf(w, w, n2);
      const __nv_bfloat16 hi = __float2bfloat16(w);
      w_hi[wrow + c] = hi;
      w_lo[wrow + c] = __float2bfloat16(w - __bfloat162float(hi));
    }
  }
  n2 = warp_sum(n2);
  if (lane == 0) wnorm[(size_t)bh * GP + g] = sqrtf(n2);
}

// ---------------------------------------------------------------------------
// Tensor-core assignment fused with the per-segment centroid sums of the next update.
// Work: segments of kSeg 128-row tiles of one head (the last segment of a head may be
// shorter), numbered head-major; CTA c takes a contiguous, balanced run of segments, so
// every segment is processed whole by one CTA and its sums do not depend on the grid or
// on how many heads the call holds.  Roles (448 threads):
//   warps 0-3 / 4-7  argmin groups A / B: the tiles of even / odd running index, one row
//               per thread (TMEM lane): argmin and runner-up of bias_g - 2 s_g over all
//               groups, ||x||^2 from the X tile, the label, the certification (a row whose
//               runner-up is within twice the error bound goes to the exact re-check), the
//               group count and the row's one in the group's one-hot tile
//   warp 8      lane 0 issues the MMAs: scores S = X [w_hi w_lo]^T into the group's TMEM
//               buffer, and, once a tile's one-hot rows are written, onehot^T X into the
//               TMEM sum buffer of the tile's segment (two buffers, by segment parity)
//   warp 9      lane 0 loads the X tiles (two TMA boxes of 128 rows x 64 columns per 128
//               columns, 128B-swizzled) into an XS-deep ring
//   warps 10-13 flush a finished segment: its sums (TMEM lane = group) and counts go to the
//               segment's slot, compacted to the groups that occur in it, and the number of
//               its uncertified rows (listed from the segment's first row on in flag_rows)
//               to flag_seg
// A CTA whose run crosses a head drains the pipeline there and loads the next head's
// weights.  Slot layout: int map[GP] (row of group g in the slot, -1 if absent), int
// cnt[GP], float rows[...][D].
// ---------------------------------------------------------------------------
namespace kma {
constexpr int NT = 448;
constexpr int NARG = 256;    // argmin threads (two groups of 128)
constexpr int MMA_WARP = 8;
constexpr int LOAD_WARP = 9;
constexpr int FL_WARP0 = 10; // flusher warps 10-13
constexpr int kXSMax = 6;
template <int D>
struct Cfg {
  static constexpr int XS = D == 64 ? 6 : 3;   // X ring depth
};
struct Bars {
  uint64_t xfull[kXSMax], xempty[kXSMax], tfull[2], tempty[2], ohfull[2], ohempty[2], sumfull[2], sumfree[2],
      cntready[2], cntfree[4];
};
}  // namespace kma

__host__ __device__ inline size_t kmeans_slot_bytes(int GP, int D) { return (size_t)GP * 8 + (size_t)GP * D * 4; }

template <int D>
__global__ void __launch_bounds__(kma::NT, 1)
    k_assign_seg(const __grid_constant__ CUtensorMap tmx, int N, int GP, int T, int SPH, int nseg,
                 const __nv_bfloat16* __restrict__ w_hi, const __nv_bfloat16* __restrict__ w_lo,
                 const float* __restrict__ bias, const float* __restrict__ wnorm, int* __restrict__ labels,
                 int* __restrict__ trace, int* __restrict__ flag_seg, int* __restrict__ flag_rows,
                 unsigned char* __restrict__ slots, float* __restrict__ xnorm, int xnorm_store, int* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = su32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) set_error(err, DERR_INDEX);
    return;
  }
  // this CTA's run of segments
  const int q = nseg / (int)gridDim.x, rem = nseg % (int)gridDim.x, c = blockIdx.x;
  const int s_begin = c * q + min(c, rem), s_end = s_begin + q + (c < rem ? 1 : 0);
  if (s_begin >= s_end) return;
  constexpr int XS = kma::Cfg<D>::XS;
  constexpr int CPR = D / 8;
  constexpr uint32_t kX = 128u * D * 2u;      // X tile
  constexpr uint32_t kOH = 128u * 128u * 2u;  // one-hot tile [2 halves][128 rows][64 groups]
  const uint32_t kW = (uint32_t)GP * D * 2u;
  const uint32_t sX = base, sOH = base + XS * kX, sWh = sOH + 2 * kOH, sWl = sWh + kW;
  float* sBias = reinterpret_cast<float*>(smem + XS * kX + 2 * kOH + 2 * kW);   // [GP]
  int* sCnt = reinterpret_cast<int*>(sBias + GP);                                // [4][GP]
  int* flw = sCnt + 4 * GP;                                                       // [2][4]
  int* sFlag = flw + 8;                                                           // [4] flagged rows per segment
  static_assert(sizeof(kma::Bars) % 8 == 0, "barrier alignment");
  kma::Bars* bars = reinterpret_cast<kma::Bars*>(sFlag + 4);
  int* sMisc = reinterpret_cast<int*>(bars + 1);   // [0] tmem, [1] abort, [2] max ||w|| bits
  volatile int* abort_flag = sMisc + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t slot_bytes = kmeans_slot_bytes(GP, D);

  if (tid == 0) {
    sMisc[1] = 0;
    for (int b = 0; b < XS; ++b) {
      mbar_init(su32(&bars->xfull[b]), 1);
      mbar_init(su32(&bars->xempty[b]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(su32(&bars->tfull[b]), 1);
      mbar_init(su32(&bars->tempty[b]), 128);
      mbar_init(su32(&bars->ohfull[b]), 128);
      mbar_init(su32(&bars->ohempty[b]), 1);
      mbar_init(su32(&bars->sumfull[b]), 1);
      mbar_init(su32(&bars->sumfree[b]), 128);
      mbar_init(su32(&bars->cntready[b]), 1);
    }
    for (int b = 0; b < 4; ++b) mbar_init(su32(&bars->cntfree[b]), 128);
    fence_barrier_init();
  }
  if (warp == kma::MMA_WARP) {
    tc_alloc(su32(&sMisc[0]), 512);
    tc_relinquish();
  }
  // both one-hot tiles start all zero (each row then only moves its one); counts zero
  for (int e = tid; e < (int)(2 * kOH / 16); e += kma::NT)
    *reinterpret_cast<uint4*>(smem + XS * kX + 16 * e) = make_uint4(0u, 0u, 0u, 0u);
  for (int e = tid; e < 4 * GP; e += kma::NT) sCnt[e] = 0;
  if (tid < 4) sFlag[tid] = 0;
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];   // scores: columns [0, 256); sums: [256, 512)
  const uint32_t IDS = idesc_bf16(128, GP, false);
  constexpr uint32_t IDA = idesc_bf16_mn(128, D, true, true);
  // error bound of one score: 2 |x.w_hi + x.w_lo - x.w| <= 2 (2^-18 + 2 D 2^-24) ||x|| ||w||
  const float kc = 2.f * (3.814697265625e-06f + 2.f * D * 5.9604644775390625e-08f);
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  int it = 0, sgi = 0;          // running tile / segment counters of this CTA (same in every role)
  bool ok = true;
  int prev_c = -1;              // argmin thread: chunk of its row's one in its group's one-hot tile
  for (int gs = s_begin; gs < s_end && ok;) {
    const int bh = gs / SPH;
    const int ge = min(s_end, (bh + 1) * SPH);            // segments [gs, ge) of head bh
    const int t_lo = (gs - bh * SPH) * kKmeansSeg, t_hi = min(T, (ge - bh * SPH) * kKmeansSeg);
    const int ntile = t_hi - t_lo;
    const size_t head = (size_t)bh * N;
    // ---- this head's weights (every role is idle here)
    for (int e = tid; e < GP * CPR; e += kma::NT) {
      const int r = e / CPR, cc = e - r * CPR;
      const size_t off = ((size_t)bh * GP + r) * D + cc * 8;
      cp_async16(sWh + tile_off(r, cc, GP), w_hi + off, true);
      cp_async16(sWl + tile_off(r, cc, GP), w_lo + off, true);
    }
    float wm = 0.f;
    for (int g = tid; g < GP; g += kma::NT) {
      sBias[g] = bias[(size_t)bh * GP + g];
      wm = fmaxf(wm, wnorm[(size_t)bh * GP + g]);
    }
    wm = warp_max(wm);
    if (tid == 0) sMisc[2] = 0;
    cp_async_wait_all();
    fence_proxy_async();
    __syncthreads();
    if (lane == 0) atomicMax(&sMisc[2], __float_as_int(wm));   // non-negative floats order as ints
    __syncthreads();
    const float wmax = __int_as_float(sMisc[2]);
    const int first = it, sg0 = sgi;   // running indices of this run's first tile / segment
    // running segment index of the run's tile n (n - first = tile offset in the run)
    auto seg_of = [&](int n) -> int { return sg0 + (t_lo + (n - first)) / kKmeansSeg - t_lo / kKmeansSeg; };

    if (warp == kma::LOAD_WARP) {
      // ---------------- loads (rows past this head's N belong to the next head or read as
      // zeros; their labels and one-hot rows are never used) ----------------
      if (lane == 0) {
        for (int n = first; n < first + ntile && ok; ++n) {
          const int xb = n % XS, n0 = (t_lo + n - first) * 128;
          if (n >= XS) ok = wait(bars->xempty[xb], ((n / XS) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(su32(&bars->xfull[xb]), kX);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_2d(sX + xb * kX + h * 16384, &tmx, 64 * h, (int)(head + n0), su32(&bars->xfull[xb]));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    } else if (warp == kma::MMA_WARP) {
      // ---------------- MMA: scores and sums issued as their inputs become ready ----------
      if (lane == 0) {
        const int last = first + ntile;
        int ns = first, nm = first;   // next tile to score / to sum
        const uint64_t t_start = gtimer();
        while (ok && nm < last) {
          bool moved = false;
          if (ns < last) {
            const int b = ns & 1, xb = ns % XS;
            if (mbar_test(su32(&bars->xfull[xb]), (ns / XS) & 1) &&
                (ns < 2 || mbar_test(su32(&bars->tempty[b]), ((ns >> 1) - 1) & 1))) {
              tc_fence_after();
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
                const uint32_t ow = (k >> 2) * (GP * 128) + (k & 3) * 32;
                tc_mma(tmem + 128 * b, sdesc(sX + xb * kX + ox, 16, 1024), sdesc(sWh + ow, 16, 1024), IDS,
                       k > 0 ? 1u : 0u);
              }
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
                const uint32_t ow = (k >> 2) * (GP * 128) + (k & 3) * 32;
                tc_mma(tmem + 128 * b, sdesc(sX + xb * kX + ox, 16, 1024), sdesc(sWl + ow, 16, 1024), IDS, 1u);
              }
              tc_commit(su32(&bars->tfull[b]));
              ++ns;
              moved = true;
            }
          }
          if (nm < ns) {
            const int b = nm & 1, xj = nm % XS;
            const int tl = t_lo + nm - first;                 // tile index in the head
            const bool seg_first = (tl % kKmeansSeg) == 0, seg_last = (tl % kKmeansSeg) == kKmeansSeg - 1 || tl == T - 1;
            const int si = seg_of(nm), sb = si & 1;
            if (mbar_test(su32(&bars->ohfull[b]), (nm >> 1) & 1) &&
                (!seg_first || si < 2 || mbar_test(su32(&bars->sumfree[sb]), ((si >> 1) - 1) & 1))) {
              tc_fence_after();
              const uint32_t tSum = tmem + 256 + 128 * sb;
#pragma unroll
              for (int k = 0; k < 8; ++k)
                tc_mma(tSum, sdesc(sOH + b * kOH + k * 2048, 16384, 1024), sdesc(sX + xj * kX + k * 2048, 16384, 1024),
                       IDA, (!seg_first || k > 0) ? 1u : 0u);
              tc_commit(su32(&bars->xempty[xj]));
              tc_commit(su32(&bars->ohempty[b]));
              if (seg_last) {
                tc_commit(su32(&bars->sumfull[sb]));
                // every count of the segment was made before its tiles' one-hot arrivals,
                // which this thread has waited for: hand them to the flusher
                mbar_arrive(su32(&bars->cntready[sb]));
              }
              ++nm;
              moved = true;
            }
          }
          if (!moved) {
            if (*abort_flag) ok = false;
            else if (gtimer() - t_start > kTimeoutNs) {
              *abort_flag = 1;
              set_error(err, DERR_WAIT_TIMEOUT);
              ok = false;
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    } else if (warp >= kma::FL_WARP0) {
      // ---------------- flusher: one thread per group (TMEM lane) ----------------
      const int r = 32 * (warp & 3) + lane;
      const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
      for (int si = sg0; si < sg0 + (ge - gs) && ok; ++si) {
        const int sb = si & 1;
        // all four flusher warps agree before their prefix barrier below
        ok = bar_and(2, 128, wait(bars->sumfull[sb], (si >> 1) & 1) && wait(bars->cntready[sb], (si >> 1) & 1));
        if (!ok) break;
        tc_fence_after();
        int* cnt4 = sCnt + (si & 3) * GP;
        const int cnt = r < GP ? cnt4[r] : 0;
        const bool occ = cnt > 0;
        const unsigned bal = __ballot_sync(0xffffffffu, occ);
        int* fl = flw + (si & 1) * 4;
        // warps in TMEM-lane order: the compacted rows follow the group order
        if (lane == 0) fl[warp & 3] = __popc(bal);
        named_sync(2, 128);
        int idx = __popc(bal & ((1u << lane) - 1u));
        for (int w = 0; w < (warp & 3); ++w) idx += fl[w];
        unsigned char* slot = slots + (size_t)(gs + si - sg0) * slot_bytes;
        int* smap = reinterpret_cast<int*>(slot);
        int* scnt = smap + GP;
        float* srow = reinterpret_cast<float*>(scnt + GP);
        if (r < GP) {
          smap[r] = occ ? idx : -1;
          scnt[r] = cnt;
        }
        const uint32_t tSum = tmem + 256 + 128 * sb;
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t v[32];
          tc_ld32(tSum + lane_off + cb, v);
          if (occ) {
            float* dst = srow + (size_t)idx * D + cb;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                                __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
        if (r < GP) cnt4[r] = 0;
        if (r == 0) {
          flag_seg[gs + si - sg0] = sFlag[si & 3];
          sFlag[si & 3] = 0;
        }
        mbar_arrive(su32(&bars->cntfree[si & 3]));   // the count buffers may take segment si + 4
        tc_fence_before();
        mbar_arrive(su32(&bars->sumfree[sb]));
      }
    } else {
      // ---------------- argmin groups (warps 0-3: even tiles, 4-7: odd tiles) ----------
      const int grp = warp >> 2;
      const int r = 32 * (warp & 3) + lane;   // row = TMEM lane
      int cnt_seg = sg0 - 1;                  // last segment whose count buffer this thread checked
      const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
      for (int n = first + ((first & 1) != grp ? 1 : 0); n < first + ntile && ok; n += 2) {
        const int b = grp, xb = n % XS;
        // scores ready; the X tile (read below for ||x||) completed before them
        ok = __all_sync(0xffffffffu, wait(bars->tfull[b], (n >> 1) & 1) && wait(bars->xfull[xb], (n / XS) & 1));
        if (!ok) break;
        const int tl = t_lo + n - first, row = tl * 128 + r;
        const bool in = row < N;
        // ||x||^2: computed from the tile by the first pass of a k-means and kept; later passes
        // read it (the load goes out before the scores are read)
        float xx = 0.f;
        if (!xnorm_store && in) xx = xnorm[head + row];
        tc_fence_after();
        // argmin and runner-up of bias_g - 2 s_g, in four interleaved sets (columns in order,
        // so the lower group wins a tie inside a set; sets merged in group order below)
        float bst[4], snd[4];
        int bix[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) { bst[u] = __int_as_float(0x7f800000); snd[u] = bst[u]; bix[u] = 0; }
        const uint64_t m2 = f2pack(-2.f, -2.f);
        for (int cb = 0; cb < GP; cb += 32) {
          uint32_t v[32];
          tc_ld32(tmem + 128 * b + lane_off + cb, v);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float sc2[2];
            f2unpack(ffma2(m2, f2pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                           f2pack(sBias[cb + e], sBias[cb + e + 1])), sc2[0], sc2[1]);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int qq = (e + u) & 3;
              const float sc = sc2[u];
              snd[qq] = fminf(snd[qq], fmaxf(bst[qq], sc));
              bix[qq] = sc < bst[qq] ? cb + e + u : bix[qq];
              bst[qq] = fminf(bst[qq], sc);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(su32(&bars->tempty[b]));
        float best = bst[0], second = snd[0];
        int bi = bix[0];
#pragma unroll
        for (int u = 1; u < 4; ++u) {
          const bool take = bst[u] < best || (bst[u] == best && bix[u] < bi);
          second = take ? fminf(best, snd[u]) : fminf(second, bst[u]);
          if (take) { best = bst[u]; bi = bix[u]; }
        }
        if (xnorm_store) {
#pragma unroll
          for (int cc = 0; cc < CPR; ++cc) {
            const uint4 u4 = *reinterpret_cast<const uint4*>(smem + xb * kX + tile_off(r, cc, 128));
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 fl = __bfloat1622float2(h2[e]);
              xx = fmaf(fl.x, fl.x, fmaf(fl.y, fl.y, xx));
            }
          }
          if (in) xnorm[head + row] = xx;
        }
        bool certified = true;
        if (in) {
          const float bound = kc * sqrtf(xx) * wmax + 1e-6f * (fabsf(best) + fabsf(second));
          labels[head + row] = bi;
          certified = second - best > 2.f * bound;
          if (certified && trace) trace[head + row] = bi;
        }
        // the one-hot tile of this group is free once the sums of its tile n - 2 are done
        if (n >= 2) ok = __all_sync(0xffffffffu, wait(bars->ohempty[b], ((n >> 1) - 1) & 1));
        if (!ok) break;
        // the count buffers of segment si were last used by segment si - 4: wait for its flush
        const int si = seg_of(n);
        if (si != cnt_seg) {
          if (si >= 4) ok = __all_sync(0xffffffffu, wait(bars->cntfree[si & 3], ((si >> 2) - 1) & 1));
          if (!ok) break;
          cnt_seg = si;
        }
        {
          // one count update per distinct label of the warp
          const unsigned peers = __match_any_sync(0xffffffffu, in ? bi : -1);
          if (in && lane == __ffs(peers) - 1) atomicAdd(&sCnt[(si & 3) * GP + bi], __popc(peers));
        }
        // uncertified: onto the segment's list for the exact re-check
        if (in && !certified)
          flag_rows[head + (size_t)(tl / kKmeansSeg) * (kKmeansSeg * 128) + atomicAdd(&sFlag[si & 3], 1)] = row;
        const int c_new = in ? (bi >> 3) : -1;
        const uint32_t oh = XS * kX + b * kOH;
        if (prev_c >= 0 && prev_c != c_new)
          *reinterpret_cast<uint4*>(smem + oh + tile_off(r, prev_c, 128)) = make_uint4(0u, 0u, 0u, 0u);
        if (c_new >= 0) {
          uint4 v4 = make_uint4(0u, 0u, 0u, 0u);
          const uint32_t one = 0x3F80u << (16 * (bi & 1));   // bf16 1.0 in the low or high half
          const int wd = (bi & 7) >> 1;
          if (wd == 0) v4.x = one; else if (wd == 1) v4.y = one; else if (wd == 2) v4.z = one; else v4.w = one;
          *reinterpret_cast<uint4*>(smem + oh + tile_off(r, c_new, 128)) = v4;
        }
        prev_c = c_new;
        fence_proxy_async();
        mbar_arrive(su32(&bars->ohfull[b]));
      }
    }
    it = first + ntile;
    sgi = sg0 + (ge - gs);
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    gs = ge;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kma::MMA_WARP) tc_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Exact re-assignment of the uncertified rows: y = A x (fp32, sequential over c),
// dist_g = sum_c (y_c - nu_gc)^2 (sequential fp32 fma over c), argmin with ties to the
// lowest g.  A row whose exact label differs from its provisional one is appended to the
// correction list (row, provisional, final) used by the next centroid update.  A and the centroids are staged in shared memory (padded rows); one warp per
// row.  grid = (RC_PER_HEAD, BH), block = 512.
// ---------------------------------------------------------------------------
constexpr int RC_PER_HEAD = 8;

template <int DT>
__global__ void __launch_bounds__(512) k_assign_recheck(const __nv_bfloat16* __restrict__ X, int N, int d,
                                                       const float* __restrict__ A, size_t a_head, int sj, int sc,
                                                       float a_scale, int D, const float* __restrict__ nu, int G,
                                                       const int* __restrict__ flag_seg, int SPH,
                                                       const int* __restrict__ flag_rows, int* __restrict__ labels,
                                                       int* __restrict__ trace, int* __restrict__ corr_count,
                                                       int4* __restrict__ corr) {
  extern __shared__ __align__(16) float sr[];
  const int bh = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float* sA = sr;                       // [D][d + 1]
  float* sNu = sA + D * (d + 1);        // [G][DT + 1]
  float* sx = sNu + G * (DT + 1);       // [16][d]
  float* sy = sx + 16 * d;              // [16][DT]
  int* pre = reinterpret_cast<int*>(sy + 16 * DT);   // [SPH + 1] first flagged item of each segment
  // the head's uncertified rows: segment s lists flag_seg[s] of them from row s * kSeg * 128 on
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int sgm = 0; sgm < SPH; ++sgm) {
      pre[sgm] = acc;
      acc += flag_seg[(size_t)bh * SPH + sgm];
    }
    pre[SPH] = acc;
  }
  __syncthreads();
  const int cnt = pre[SPH];
  if ((int)blockIdx.x * 16 >= cnt) return;
  const size_t head = (size_t)bh * N;
  const float* Ah = A + a_head * bh;
  const float* nuh = nu + (size_t)bh * G * DT;
  // staging loops unrolled so that each thread keeps several loads in flight (A's
  // unit-stride index fastest)
  if (sj == 1) {
#pragma unroll 8
    for (int e = threadIdx.x; e < D * d; e += 512) {
      const int c = e / D, j = e - c * D;
      sA[j * (d + 1) + c] = Ah[(size_t)j + (size_t)c * sc];
    }
  } else {
#pragma unroll 8
    for (int e = threadIdx.x; e < D * d; e += 512) {
      const int j = e / d, c = e - j * d;
      sA[j * (d + 1) + c] = Ah[(size_t)j * sj + (size_t)c * sc];
    }
  }
#pragma unroll 8
  for (int e = threadIdx.x; e < G * DT; e += 512) {
    const int g = e / DT, c = e - g * DT;
    sNu[g * (DT + 1) + c] = nuh[e];
  }
  __syncthreads();
  float* wx = sx + warp * d;
  float* wy = sy + warp * DT;
  for (int i = blockIdx.x * 16 + warp; i < cnt; i += gridDim.x * 16) {
    int lo = 0, hi = SPH - 1;   // segment of item i: the last with pre[s] <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int row = flag_rows[head + (size_t)lo * (kKmeansSeg * 128) + (i - pre[lo])];
    if (row < 0 || row >= N) continue;
    for (int c = lane; c < d; c += 32) wx[c] = bf2f(X[(head + row) * d + c]);
    __syncwarp();
    for (int j = lane; j < DT; j += 32) {
      float acc = 0.f;
      if (j < D) {
        for (int c = 0; c < d; ++c) acc = fmaf(wx[c], sA[j * (d + 1) + c], acc);
        acc *= a_scale;
      }
      wy[j] = acc;
    }
    __syncwarp();
    float best = __int_as_float(0x7f800000);
    int bi = 0x7fffffff;
    for (int g = lane; g < G; g += 32) {
      const float* mu = sNu + g * (DT + 1);
      float dist = 0.f;
      for (int c = 0; c < DT; ++c) {
        const float t = wy[c] - mu[c];
        dist = fmaf(t, t, dist);
      }
      if (dist < best) { best = dist; bi = g; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob < best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (lane == 0) {
      const int prov = labels[head + row];
      if (prov != bi) {
        // the row entered the pass's sums under its provisional label
        const int slot = atomicAdd(&corr_count[bh], 1);
        if (slot < N) corr[head + slot] = make_int4(row, prov, bi, 0);
      }
      labels[head + row] = bi;
      if (trace) trace[head + row] = bi;
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Cell mass on the tensor cores.  p(a, g) = mean over the queries q of group a of
// softmax_g(z_q[g] + ln n_g) over non-empty K/V groups, z_q = s q . c_g.
// c_g is split into three bf16 parts (c = c1 + c2 + c3 to ~2^-24), so the products with
// the exact bf16 q are exact and z carries only fp32 accumulation error.
// One CTA = one head x a run of query groups; every group's permuted rows are gathered
// through perm_q in 128-row tiles; column sums run over rows in fixed order, so the
// result is deterministic.  grid = (CTAS_PER_HEAD, BH), block = 128.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_split3(const float* __restrict__ C, int G, int GP, int d,
                                               __nv_bfloat16* __restrict__ c1, __nv_bfloat16* __restrict__ c2,
                                               __nv_bfloat16* __restrict__ c3) {
  const int g = blockIdx.x, bh = blockIdx.y;
  for (int c = threadIdx.x; c < d; c += 128) {
    const float x = g < G ? C[((size_t)bh * G + g) * d + c] : 0.f;
    const __nv_bfloat16 a = __float2bfloat16(x);
    const float r1 = x - __bfloat162float(a);
    const __nv_bfloat16 b = __float2bfloat16(r1);
    const __nv_bfloat16 e = __float2bfloat16(r1 - __bfloat162float(b));
    const size_t o = ((size_t)bh * GP + g) * d + c;
    c1[o] = a;
    c2[o] = b;
    c3[o] = e;
  }
}

// Roles of the 576 threads of the persistent cell-mass kernel: warps 0-15 take the softmax
// of tile row r = TMEM lane r, split over four column quarters (warps w, w+4, w+8, w+12):
// each quarter exponentiates against its own running max, the quarters exchange (max, sum)
// once, scale, and reduce their columns over the warp's 32 rows with a fixed butterfly;
// warp 16 allocates TMEM and its lane 0 issues the MMAs, warp 17 gathers the tile's query
// rows through perm_q (cp.async) into a two-deep ring.  CTA b takes the (head, query group) items [b per, (b+1) per) in order;
// the K/V centroid parts of a head are reloaded when the head changes.
namespace cmk {
constexpr int NT = 576;
constexpr int NSM = 512;   // softmax threads
constexpr int MMA_WARP = 16;
constexpr int LOAD_WARP = 17;
struct Bars {
  uint64_t xfull[2], xempty[2], tfull[2], tempty[2], mready[2], pready[2];
};
}  // namespace cmk

// Sum over the 32 lanes of each of the 32 columns in v[]: afterwards lane l holds, in v[0],
// the sum of column l (butterfly reduce-scatter; fixed order, so deterministic).
__device__ __forceinline__ float lane_column_sum32(float* v, int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int k = 0; k < w; ++k) {
      const float send = upper ? v[k] : v[k + w];
      const float keep = upper ? v[k + w] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

template <int D>
__global__ void __launch_bounds__(cmk::NT, 1) k_cell_mass_tc(const __nv_bfloat16* __restrict__ Q, int N, int Gq,
                                                            int Gk, int GP, int nitems,
                                                            const int* __restrict__ perm_q,
                                                            const int* __restrict__ qoff,
                                                            const int* __restrict__ koff,
                                                            const __nv_bfloat16* __restrict__ c1,
                                                            const __nv_bfloat16* __restrict__ c2,
                                                            const __nv_bfloat16* __restrict__ c3, float scale_log2,
                                                            const int* __restrict__ frame_id,
                                                            const int* __restrict__ visk, int F,
                                                            float* __restrict__ mass, int* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = su32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) set_error(err, DERR_INDEX);
    return;
  }
  const int per = (nitems + gridDim.x - 1) / gridDim.x;
  const int i0 = blockIdx.x * per, i1 = min(nitems, i0 + per);
  if (i0 >= i1) return;
  constexpr uint32_t kX = 128u * D * 2u;
  constexpr int CPR = D / 8;
  const uint32_t kC = (uint32_t)GP * D * 2u;
  const uint32_t sX = base, sC = base + 2 * kX;
  float* part = reinterpret_cast<float*>(smem + 2 * kX + 3 * kC);   // [2 tiles][16 warps][32]
  float2* msx = reinterpret_cast<float2*>(part + 2 * 16 * 32);       // [2 tiles][4 quarters][128]
  float* colacc = reinterpret_cast<float*>(msx + 2 * 4 * 128);       // [GP]
  float* lnn = colacc + GP;                                          // [GP] log2 n_g or -inf
  cmk::Bars* bars = reinterpret_cast<cmk::Bars*>(lnn + GP);
  int* sMisc = reinterpret_cast<int*>(bars + 1);                     // [0] tmem, [1] abort
  // frame-causal: [F][GP + 1] log2 of the keys of g a frame-f query sees, or -inf
  float* lnf = reinterpret_cast<float*>(sMisc + 4);
  const bool causal = frame_id != nullptr;
  volatile int* abort_flag = sMisc + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG_INF = __int_as_float(0xff800000);

  if (tid == 0) {
    sMisc[1] = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(su32(&bars->xfull[b]), 32);
      mbar_init(su32(&bars->xempty[b]), 1);
      mbar_init(su32(&bars->tfull[b]), 1);
      mbar_init(su32(&bars->tempty[b]), cmk::NSM);
      mbar_init(su32(&bars->mready[b]), cmk::NSM);
      mbar_init(su32(&bars->pready[b]), cmk::NSM);
    }
    fence_barrier_init();
  }
  if (warp == cmk::MMA_WARP) {
    tc_alloc(su32(&sMisc[0]), 256);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];
  const uint32_t idesc = idesc_bf16(128, GP, false);
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  int tile = 0;   // running tile counter of this role (identical across roles)
  bool ok = true;
  for (int seg0 = i0; seg0 < i1 && ok;) {
    const int bh = seg0 / Gq;
    const int seg1 = min(i1, (bh + 1) * Gq);
    const size_t head = (size_t)bh * N;
    const int* qo = qoff + (size_t)bh * (Gq + 1);
    // ---- this head's centroid parts and log2 group sizes (every role is idle here)
    __syncthreads();
    for (int e = tid; e < GP * CPR; e += cmk::NT) {
      const int r = e / CPR, c = e - r * CPR;
      const size_t off = ((size_t)bh * GP + r) * D + c * 8;
      const uint32_t o = tile_off(r, c, GP);
      cp_async16(sC + o, c1 + off, true);
      cp_async16(sC + kC + o, c2 + off, true);
      cp_async16(sC + 2 * kC + o, c3 + off, true);
    }
    for (int g = tid; g < GP; g += cmk::NT) {
      const int n = g < Gk ? koff[(size_t)bh * (Gk + 1) + g + 1] - koff[(size_t)bh * (Gk + 1) + g] : 0;
      lnn[g] = n > 0 ? log2f((float)n) : NEG_INF;
      colacc[g] = 0.f;
    }
    if (causal) {
      for (int e = tid; e < F * GP; e += cmk::NT) {
        const int f = e / GP, g = e - f * GP;
        const int n = g < Gk ? visk[((size_t)bh * Gk + g) * F + f] : 0;
        lnf[f * (GP + 1) + g] = n > 0 ? log2f((float)n) : NEG_INF;
      }
    }
    cp_async_wait_all();
    fence_proxy_async();
    __syncthreads();
    const int a0 = seg0 - bh * Gq, a1 = seg1 - bh * Gq;

    if (warp == cmk::LOAD_WARP) {
      // ---------------- gather ----------------
      for (int a = a0; a < a1 && ok; ++a) {
        for (int t0 = qo[a]; t0 < qo[a + 1]; t0 += 128, ++tile) {
          const int b = tile & 1, nr = min(128, qo[a + 1] - t0);
          // the tile's row indices: all four loads go out together, before the slot wait
          int rows4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) rows4[k] = 32 * k + lane < nr ? perm_q[head + t0 + 32 * k + lane] : -1;
          if (tile >= 2) ok = __all_sync(0xffffffffu, wait(bars->xempty[b], ((tile >> 1) - 1) & 1));
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int r = 32 * k + lane;
            int myrow = -1;
            if (r < nr) {
              myrow = rows4[k];
              if (myrow < 0 || myrow >= N) { set_error(err, DERR_INDEX); myrow = -1; }
            }
#pragma unroll
            for (int it = 0; it < CPR; ++it) {
              const int e = it * 32 + lane, rr = e / CPR, c = e % CPR;
              const int row = __shfl_sync(0xffffffffu, myrow, rr);
              cp_async16(sX + b * kX + tile_off(32 * k + rr, c, 128), Q + (head + (row < 0 ? 0 : row)) * D + c * 8,
                         row >= 0);
            }
          }
          cp_async_arrive_noinc(su32(&bars->xfull[b]));
        }
      }
      cp_async_wait_all();
    } else if (warp == cmk::MMA_WARP) {
      // ---------------- MMA ----------------
      if (lane == 0) {
        for (int a = a0; a < a1 && ok; ++a) {
          for (int t0 = qo[a]; t0 < qo[a + 1]; t0 += 128, ++tile) {
            const int b = tile & 1;
            ok = wait(bars->xfull[b], (tile >> 1) & 1) && (tile < 2 || wait(bars->tempty[b], ((tile >> 1) - 1) & 1));
            if (!ok) break;
            tc_fence_after();
            int n = 0;
            for (int part3 = 0; part3 < 3; ++part3) {
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
                const uint32_t oc = (k >> 2) * (GP * 128) + (k & 3) * 32;
                tc_mma(tmem + 128 * b, sdesc(sX + b * kX + ox, 16, 1024), sdesc(sC + part3 * kC + oc, 16, 1024),
                       idesc, n++ > 0 ? 1u : 0u);
              }
            }
            tc_commit(su32(&bars->tfull[b]));
            tc_commit(su32(&bars->xempty[b]));
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      tile = __shfl_sync(0xffffffffu, tile, 0);
    } else if (warp < 16) {
      // ---------------- softmax + column sums (warp = quarter * 4 + row group) ----------------
      const int qt = warp >> 2, rg = warp & 3;
      const int r = rg * 32 + lane;   // tile row = TMEM lane
      const int cb = qt * 32;         // this quarter's columns
      const uint32_t lane_off = (uint32_t)(rg * 32) << 16;
      for (int a = a0; a < a1 && ok; ++a) {
        const int n_a = qo[a + 1] - qo[a];
        if (n_a == 0) {
          if (qt == 0 && r < Gk) mass[((size_t)bh * Gq + a) * Gk + r] = 0.f;
          continue;
        }
        for (int t0 = qo[a]; t0 < qo[a + 1]; t0 += 128, ++tile) {
          const int b = tile & 1, nr = min(128, qo[a + 1] - t0);
          ok = __all_sync(0xffffffffu, wait(bars->tfull[b], (tile >> 1) & 1));
          if (!ok) break;
          tc_fence_after();
          float v[32];
          if (cb < GP) {
            uint32_t u[32];
            tc_ld32(tmem + 128 * b + lane_off + cb, u);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(u[e]);
          }
          tc_fence_before();
          mbar_arrive(su32(&bars->tempty[b]));
          // log2 group sizes this row sees (frame-causal: the keys of frames <= its frame)
          const float* lnrow = lnn;
          if (causal && r < nr) {
            const int row = perm_q[head + t0 + r];
            int f = (row >= 0 && row < N) ? frame_id[row] : 0;
            f = f < 0 ? 0 : (f >= F ? F - 1 : f);
            lnrow = lnf + f * (GP + 1);
          }
          // this quarter: logits in log2 units, local max and local sum
          float mq = NEG_INF;
          if (cb < GP) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float ln = lnrow[cb + e];
              v[e] = ln == NEG_INF ? NEG_INF : fmaf(v[e], scale_log2, ln);
              mq = fmaxf(mq, v[e]);
            }
          }
          float sq = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            v[e] = (cb < GP && v[e] != NEG_INF) ? ex2(v[e] - mq) : 0.f;
            sq += v[e];
          }
          msx[(b * 4 + qt) * 128 + r] = make_float2(mq, sq);
          mbar_arrive(su32(&bars->mready[b]));
          ok = __all_sync(0xffffffffu, wait(bars->mready[b], (tile >> 1) & 1));
          if (!ok) break;
          // row max and sum over the quarters (fixed order), then this quarter's scale
          float M = NEG_INF;
#pragma unroll
          for (int q = 0; q < 4; ++q) M = fmaxf(M, msx[(b * 4 + q) * 128 + r].x);
          float S = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 ms = msx[(b * 4 + q) * 128 + r];
            S += ms.x == NEG_INF ? 0.f : ms.y * ex2(ms.x - M);
          }
          const float f = (r < nr && S > 0.f && mq != NEG_INF) ? ex2(mq - M) / S : 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= f;
          part[(b * 16 + warp) * 32 + lane] = lane_column_sum32(v, lane);
          mbar_arrive(su32(&bars->pready[b]));
          ok = __all_sync(0xffffffffu, wait(bars->pready[b], (tile >> 1) & 1));
          if (!ok) break;
          if (qt == 0 && r < GP) {
            // column r: the four row groups of its quarter, in order
            const float* pb = part + (b * 16 + (r >> 5) * 4) * 32 + (r & 31);
            colacc[r] += (pb[0] + pb[32]) + (pb[64] + pb[96]);
            if (t0 + 128 >= qo[a + 1]) {
              if (r < Gk) mass[((size_t)bh * Gq + a) * Gk + r] = colacc[r] / (float)n_a;
              colacc[r] = 0.f;
            }
          }
        }
      }
    }
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    seg0 = seg1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == cmk::MMA_WARP) tc_dealloc(tmem, 256);
}

}  // namespace km

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
int kmeans_gp(int G) { return (G + 31) / 32 * 32; }

size_t assign_acc_smem(int D, int GP) {
  const int XS = D == 64 ? km::kma::Cfg<64>::XS : km::kma::Cfg<128>::XS;
  return (size_t)XS * 128 * D * 2 + 2 * (size_t)128 * 128 * 2 + 2 * (size_t)GP * D * 2 + (size_t)GP * 4 +
         (size_t)4 * GP * 4 + 12 * 4 + sizeof(km::kma::Bars) + 16;
}

KmPlan kmeans_plan(int BH, int N) {
  KmPlan pl{};
  pl.T = ceil_div(N, 128);
  pl.SPH = ceil_div(pl.T, kKmeansSeg);
  pl.nseg = BH * pl.SPH;
  pl.grid = pl.nseg < kKmeansCtas ? pl.nseg : kKmeansCtas;
  return pl;
}

size_t kmeans_slots_bytes(int BH, int N, int GP, int d) {
  return (size_t)BH * kmeans_plan(BH, N).SPH * km::kmeans_slot_bytes(GP, d);
}

cudaError_t launch_seed_rows(const void* X, int BH, int N, int d, int G, uint64_t seed, HeadMap hm, int purpose,
                             float* m, int* init_out, int* err, cudaStream_t st) {
  const size_t sm = (size_t)2 * G * 4;
  cudaFuncSetAttribute(km::k_seed_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_seed_rows<<<BH, 256, sm, st>>>((const __nv_bfloat16*)X, N, d, G, seed, hm, purpose, m, init_out, err);
  return cudaGetLastError();
}

size_t centroid_weights_smem(int d, int D, int N) {
  const int SPH = kmeans_plan(1, N).SPH;
  return (size_t)km::WG_PER_CTA * d * 8 + km::WG_PER_CTA * 4 +
         ((size_t)km::cw_scratch_floats(d, D, SPH) + (size_t)km::WG_PER_CTA * d + (size_t)km::WG_PER_CTA * 128) * 4;
}

cudaError_t launch_centroid_weights(float* m, int BH, int G, int d, const float* A, size_t a_head, int sj, int sc,
                                    float a_scale, int D, int DT, int mode, const void* slots,
                                    const int* corr_count, const void* corr, const void* X, int N, float* nu,
                                    float* bias, float* wnorm, void* w_hi, void* w_lo, int* err, cudaStream_t st) {
  const int GP = kmeans_gp(G);
  const size_t sm = centroid_weights_smem(d, D, N);
  const KmPlan pl = kmeans_plan(BH, N);
  km::KmPartials pp{(const unsigned char*)slots, corr_count, (const int4*)corr, (const __nv_bfloat16*)X, N, pl.SPH};
  cudaFuncSetAttribute(km::k_centroid_weights, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_centroid_weights<<<dim3(ceil_div(GP, km::WG_PER_CTA), BH), km::CW_THREADS, sm, st>>>(
      m, G, GP, d, A, a_head, sj, sc, a_scale, D, DT, mode, pp, nu, bias, wnorm, (__nv_bfloat16*)w_hi,
      (__nv_bfloat16*)w_lo, err);
  return cudaGetLastError();
}

cudaError_t launch_assign_acc(const void* X, int BH, int N, int d, int G, const void* w_hi, const void* w_lo,
                              const float* bias, const float* wnorm, int* labels, int* trace, int* flag_seg,
                              int* flag_rows, void* slots, float* xnorm, int xnorm_store, int* err,
                              cudaStream_t st) {
  const int GP = kmeans_gp(G);
  const size_t sm = assign_acc_smem(d, GP);
  const KmPlan pl = kmeans_plan(BH, N);
  CUtensorMap tmx;
  cudaError_t e = make_tmap_bf16_rows(&tmx, X, (unsigned long long)BH * N, d, 128);
  if (e != cudaSuccess) return e;
  if (d == 64) {
    cudaFuncSetAttribute(km::k_assign_seg<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_assign_seg<64><<<pl.grid, km::kma::NT, sm, st>>>(
        tmx, N, GP, pl.T, pl.SPH, pl.nseg, (const __nv_bfloat16*)w_hi, (const __nv_bfloat16*)w_lo, bias, wnorm,
        labels, trace, flag_seg, flag_rows, (unsigned char*)slots, xnorm, xnorm_store, err);
  } else {
    cudaFuncSetAttribute(km::k_assign_seg<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_assign_seg<128><<<pl.grid, km::kma::NT, sm, st>>>(
        tmx, N, GP, pl.T, pl.SPH, pl.nseg, (const __nv_bfloat16*)w_hi, (const __nv_bfloat16*)w_lo, bias, wnorm,
        labels, trace, flag_seg, flag_rows, (unsigned char*)slots, xnorm, xnorm_store, err);
  }
  return cudaGetLastError();
}

size_t recheck_smem(int d, int D, int DT, int G, int N) {
  return ((size_t)D * (d + 1) + (size_t)G * (DT + 1) + 16 * (size_t)d + 16 * (size_t)DT) * 4 +
         ((size_t)kmeans_plan(1, N).SPH + 1) * 4;
}

template <int DT>
static cudaError_t recheck_dt(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                              float a_scale, int D, const float* nu, int G, const int* flag_seg,
                              const int* flag_rows, int* labels, int* trace, int* corr_count, void* corr,
                              cudaStream_t st) {
  const size_t sm = recheck_smem(d, D, DT, G, N);
  const int SPH = kmeans_plan(1, N).SPH;
  cudaFuncSetAttribute(km::k_assign_recheck<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_assign_recheck<DT><<<dim3(km::RC_PER_HEAD, BH), 512, sm, st>>>((const __nv_bfloat16*)X, N, d, A, a_head, sj,
                                                                      sc, a_scale, D, nu, G, flag_seg, SPH, flag_rows,
                                                                      labels, trace, corr_count, (int4*)corr);
  return cudaGetLastError();
}

cudaError_t launch_assign_recheck(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                                  float a_scale, int D, const float* nu, int G, const int* flag_seg,
                                  const int* flag_rows, int* labels, int* trace, int* corr_count, void* corr,
                                  cudaStream_t st) {
  switch (kmeans_dt(D)) {
    case 8: return recheck_dt<8>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_seg, flag_rows, labels, trace, corr_count, corr, st);
    case 16: return recheck_dt<16>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_seg, flag_rows, labels, trace, corr_count, corr, st);
    case 32: return recheck_dt<32>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_seg, flag_rows, labels, trace, corr_count, corr, st);
    case 64: return recheck_dt<64>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_seg, flag_rows, labels, trace, corr_count, corr, st);
    case 128: return recheck_dt<128>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_seg, flag_rows, labels, trace, corr_count, corr, st);
    default: return cudaErrorInvalidValue;
  }
}

size_t cell_mass_tc_smem(int D, int GP, int F) {
  return (size_t)2 * 128 * D * 2 + 3 * (size_t)GP * D * 2 + (size_t)2 * 16 * 32 * 4 + (size_t)2 * 4 * 128 * 8 +
         (size_t)2 * GP * 4 + sizeof(km::cmk::Bars) + 16 + (size_t)F * (GP + 1) * 4;
}

static int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        n <= 0)
      n = 148;
  }
  return n;
}

cudaError_t launch_cell_mass_tc(const void* Q, int BH, int N, int d, int Gq, int Gk, const int* perm_q, const int* qoff,
                                const int* koff, const float* C, float scale, void* c1, void* c2, void* c3,
                                const Causal& cz, float* mass, int* err, cudaStream_t st) {
  const int GP = kmeans_gp(Gk);
  km::k_split3<<<dim3(GP, BH), 128, 0, st>>>(C, Gk, GP, d, (__nv_bfloat16*)c1, (__nv_bfloat16*)c2,
                                            (__nv_bfloat16*)c3);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int F = cz.on() ? cz.F : 0;
  const size_t sm = cell_mass_tc_smem(d, GP, F);
  const int nitems = BH * Gq;
  const int grid = nitems < sm_count() ? nitems : sm_count();
  const float scale_log2 = scale * 1.4426950408889634f;
  if (d == 64) {
    cudaFuncSetAttribute(km::k_cell_mass_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_cell_mass_tc<64><<<grid, km::cmk::NT, sm, st>>>((const __nv_bfloat16*)Q, N, Gq, Gk, GP, nitems, perm_q, qoff,
                                                         koff, (const __nv_bfloat16*)c1, (const __nv_bfloat16*)c2,
                                                         (const __nv_bfloat16*)c3, scale_log2, cz.frame_id, cz.visk,
                                                         F, mass, err);
  } else {
    cudaFuncSetAttribute(km::k_cell_mass_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_cell_mass_tc<128><<<grid, km::cmk::NT, sm, st>>>((const __nv_bfloat16*)Q, N, Gq, Gk, GP, nitems, perm_q,
                                                          qoff, koff, (const __nv_bfloat16*)c1,
                                                          (const __nv_bfloat16*)c2, (const __nv_bfloat16*)c3,
                                                          scale_log2, cz.frame_id, cz.visk, F, mass, err);
  }
  return cudaGetLastError();
}

}  // namespace spr
