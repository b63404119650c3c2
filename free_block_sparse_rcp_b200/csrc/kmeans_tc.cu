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
// mode 0: m holds the centroids (the seeds).
// mode 1: m_g = (sum of the rows assigned to g) / (their count): the partial sums the
//         previous assignment pass left per (CTA, head) slot, added in ascending CTA order
//         in fp64, then the label corrections of the exact re-check applied in ascending
//         row order (a row moves from its provisional group to its final one); an empty
//         group keeps its centroid.  m is updated in place.
// mode 2: as mode 1 but an empty group gets 0, the means are written to m and no weights
//         are formed (the K/V group centroids after the last pass).
// Weights, two centroids per warp: nu = A m (fp32, sequential over c), bias = ||nu||^2,
//   w = A^T nu (sequential over j) -> w_hi = bf16(w), w_lo = bf16(w - w_hi); wnorm = ||w||.
// Rows g in [G, GP) are padding: w = 0, bias = +inf.
// grid = (ceil(GP / WG_PER_CTA), BH), block = 256.
// ---------------------------------------------------------------------------
constexpr int WG_PER_CTA = 16;
constexpr int CW_THREADS = 256;

struct KmPartials {
  const float* psum;          // [grid][maxh][GP][d]
  const int* pcnt;            // [grid][maxh][GP]
  const int* corr_count;      // [BH]
  const int4* corr;           // [BH][N] (row, provisional label, final label, -)
  const __nv_bfloat16* X;     // rows
  int N, T, per, maxh, grid;
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
  float* sA = reinterpret_cast<float*>(cnt + WG_PER_CTA);    // [D][d + 1]
  float* sMg = sA + D * (d + 1);                             // [WG_PER_CTA][d] this CTA's centroids
  float* sNu = sMg + WG_PER_CTA * d;                         // [WG_PER_CTA][128] their nu
  const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g0 = blockIdx.x * WG_PER_CTA, g1 = min(GP, g0 + WG_PER_CTA);
  if (mode != 0) {
    // ---- means from the partial sums of the previous pass
    const int h0 = bh * pp.T, h1 = h0 + pp.T;
    const int b_lo = h0 / pp.per, b_hi = min(pp.grid - 1, (h1 - 1) / pp.per);
    // per element, the slots in ascending CTA order (0 + s_lo + ... + s_hi, as the definition
    // of the mean reads); the loads of all slots of an element are independent and go out
    // together
    for (int e = tid; e < WG_PER_CTA * d; e += CW_THREADS) {
      const int gi = e / d, c = e - gi * d;
      double a = 0.0;
      if (gi < g1 - g0) {
#pragma unroll 4
        for (int b = b_lo; b <= b_hi; ++b) {
          const int slot = b * pp.maxh + (bh - (b * pp.per) / pp.T);
          a += (double)pp.psum[((size_t)slot * GP + g0 + gi) * d + c];
        }
      }
      acc[e] = a;
    }
    if (tid < WG_PER_CTA) {
      int n = 0;
      if (tid < g1 - g0)
        for (int b = b_lo; b <= b_hi; ++b) n += pp.pcnt[(size_t)(b * pp.maxh + (bh - (b * pp.per) / pp.T)) * GP + g0 + tid];
      cnt[tid] = n;
    }
    __syncthreads();
    if (warp == 0) {
      // corrections in ascending row order (the list itself is in arbitrary order)
      const int nc = min(pp.corr_count[bh], pp.N);
      const int4* cl = pp.corr + (size_t)bh * pp.N;
      int last = -1;
      while (true) {
        int best = 0x7fffffff, bi = -1;
        for (int i = lane; i < nc; i += 32) {
          const int r = cl[i].x;
          if (r > last && r < best) { best = r; bi = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const int ob = __shfl_xor_sync(0xffffffffu, best, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ob < best) { best = ob; bi = oi; }
        }
        if (bi < 0) break;
        last = best;
        const int4 cr = cl[bi];
        if (cr.x < 0 || cr.x >= pp.N) { if (lane == 0) set_error(err, DERR_INDEX); break; }
        const bool from = cr.y >= g0 && cr.y < g1, to = cr.z >= g0 && cr.z < g1;
        if (from || to) {
          const __nv_bfloat16* xr = pp.X + ((size_t)bh * pp.N + cr.x) * d;
          for (int c = lane; c < d; c += 32) {
            const double x = (double)bf2f(xr[c]);
            if (from) acc[(cr.y - g0) * d + c] -= x;
            if (to) acc[(cr.z - g0) * d + c] += x;
          }
          if (lane == 0) {
            if (from) cnt[cr.y - g0] -= 1;
            if (to) cnt[cr.z - g0] += 1;
          }
        }
        __syncwarp();
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
  // staging loops unrolled so that each thread keeps several loads in flight
#pragma unroll 8
  for (int e = tid; e < D * d; e += CW_THREADS) {
    const int j = e / d, c = e - j * d;
    sA[j * (d + 1) + c] = Ah[(size_t)j * sj + (size_t)c * sc];
  }
  __syncthreads();
#pragma unroll 8
  for (int e = tid; e < WG_PER_CTA * d; e += CW_THREADS) {
    const int gi = e / d, c = e - gi * d, g = g0 + gi;
    sMg[e] = (g < g1 && g < G) ? m[((size_t)bh * G + g) * d + c] : 0.f;
  }
  __syncthreads();
  // warp w forms the weights of groups g0 + w and g0 + w + 8 together; lanes split j for
  // nu = A m and c for w = A^T nu, each sum in ascending order of its index
  static_assert(WG_PER_CTA == 2 * (CW_THREADS / 32), "two groups per warp");
  const int gl[2] = {warp, warp + 8};
  bool live[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int g = g0 + gl[u];
    live[u] = g < g1 && g < G;
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
  }
  if (!live[0] && !live[1]) return;
  float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  {
    const float* m0 = sMg + gl[0] * d;
    const float* m1 = sMg + gl[1] * d;
    for (int c = 0; c < d; ++c) {
      const float x0 = m0[c], x1 = m1[c];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int j = lane + 32 * k;
        if (j < D) {
          const float a = sA[j * (d + 1) + c];
          acc2[0][k] = fmaf(a, x0, acc2[0][k]);
          acc2[1][k] = fmaf(a, x1, acc2[1][k]);
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int g = g0 + gl[u];
    float b2 = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = lane + 32 * k;
      if (j < D) {
        const float a = acc2[u][k] * a_scale;
        sNu[gl[u] * 128 + j] = a;
        b2 = fmaf(a, a, b2);
      }
    }
    b2 = warp_sum(b2);
    if (live[u]) {
      for (int j = lane; j < DT; j += 32) nu[((size_t)bh * G + g) * DT + j] = j < D ? sNu[gl[u] * 128 + j] : 0.f;
      if (lane == 0) bias[(size_t)bh * GP + g] = b2;
    }
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 2; ++u)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc2[u][k] = 0.f;
  {
    const float* n0 = sNu + gl[0] * 128;
    const float* n1 = sNu + gl[1] * 128;
    for (int j = 0; j < D; ++j) {
      const float y0 = n0[j], y1 = n1[j];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        if (c < d) {
          const float a = sA[j * (d + 1) + c];
          acc2[0][k] = fmaf(a, y0, acc2[0][k]);
          acc2[1][k] = fmaf(a, y1, acc2[1][k]);
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int g = g0 + gl[u];
    const size_t wrow = ((size_t)bh * GP + g) * d;
    float n2 = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = lane + 32 * k;
      if (c < d) {
        const float w = a_scale * acc2[u][k];
        n2 = fmaf(w, w, n2);
        if (live[u]) {
          const __nv_bfloat16 hi = __float2bfloat16(w);
          w_hi[wrow + c] = hi;
          w_lo[wrow + c] = __float2bfloat16(w - __bfloat162float(hi));
        }
      }
    }
    n2 = warp_sum(n2);
    if (live[u] && lane == 0) wnorm[(size_t)bh * GP + g] = sqrtf(n2);
  }
}

// ---------------------------------------------------------------------------
// Tensor-core assignment fused with the centroid sums of the next update.
// Persistent: CTA b takes the global 128-row tiles [b per, (b+1) per) (tile i = row tile
// i mod T of head i / T) and runs them through a pipeline:
//   warp 19     (lane 0) loads the X tile (contiguous rows, two TMA boxes of 128 rows x 64
//               columns, 128B-swizzled) into a three-deep ring
//   warp 18     (lane 0) scores S = X [w_hi w_lo]^T into a double-buffered TMEM tile, then,
//               once the labels are known, adds onehot(labels)^T X into a TMEM sum
//               (M = 128 groups x N = d; A and B both MN-major, read straight from the
//               one-hot tile and the X tile)
//   warps 0-15  row r = TMEM lane r, columns split in four quarters (warps w, w + 4, w + 8,
//               w + 12): argmin and runner-up of bias_g - 2 s_g per quarter and the
//               quarter's ||x||^2, handed over through shared memory (double-buffered)
//   warps 16-17 the finisher, two rows per thread: merges the quarters, writes the label
//               and the count, puts a row whose runner-up is within twice the error bound
//               on the list of the exact re-check (which corrects its label and, through
//               the correction list, the sums), and writes the tile's one-hot rows.  The
//               argmin warps go on to the next tile meanwhile.
// When the CTA leaves a head (or ends) the sums and the per-group counts go to the
// partial slot (CTA, head - first head of the CTA).
// ---------------------------------------------------------------------------
namespace kma {
constexpr int NT = 640;
constexpr int NEPI = 512;   // argmin threads (warps 0-15)
constexpr int NFIN = 64;    // finisher threads (warps 16-17), two rows each
constexpr int NQ = 4;   // column quarters
constexpr int FIN_WARP = 16;
constexpr int MMA_WARP = 18;
constexpr int LOAD_WARP = 19;
constexpr int XS = 3;   // X ring depth
struct Bars {
  uint64_t xfull[XS], xempty[XS], tfull[2], tempty[2], ohfull, ohempty, sumdone, xready[2], xfree[2], epidone;
};
struct Half {
  float best, second, xx;
  int bi;
};
}  // namespace kma

template <int D>
__global__ void __launch_bounds__(kma::NT, 1)
    k_assign_acc(const __grid_constant__ CUtensorMap tmx, int N, int GP, int T, int total, int per, int maxh,
                 const __nv_bfloat16* __restrict__ w_hi, const __nv_bfloat16* __restrict__ w_lo,
                 const float* __restrict__ bias, const float* __restrict__ wnorm, int* __restrict__ labels,
                 int* __restrict__ trace, int* __restrict__ flag_count, int* __restrict__ flag_rows,
                 float* __restrict__ psum, int* __restrict__ pcnt, int* err) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = su32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) set_error(err, DERR_INDEX);
    return;
  }
  const int t0 = blockIdx.x * per, t1 = min(total, t0 + per);
  if (t0 >= t1) return;
  constexpr int CPR = D / 8;
  constexpr uint32_t kX = 128u * D * 2u;      // X tile
  constexpr uint32_t kOH = 128u * 128u * 2u;  // one-hot tile [2 halves][128 rows][64 groups]
  const uint32_t kW = (uint32_t)GP * D * 2u;
  constexpr int XS = kma::XS;
  const uint32_t sX = base, sOH = base + XS * kX, sWh = sOH + kOH, sWl = sWh + kW;
  kma::Half* xchg = reinterpret_cast<kma::Half*>(smem + XS * kX + kOH + 2 * kW);   // [2 tiles][NQ][128]
  float* sBias = reinterpret_cast<float*>(xchg + 2 * kma::NQ * 128);                // [GP]
  int* sCnt = reinterpret_cast<int*>(sBias + GP);                                    // [GP]
  kma::Bars* bars = reinterpret_cast<kma::Bars*>(sCnt + GP);
  int* sMisc = reinterpret_cast<int*>(bars + 1);   // [0] tmem, [1] abort, [2] max ||w|| bits
  volatile int* abort_flag = sMisc + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    sMisc[1] = 0;
    for (int b = 0; b < XS; ++b) {
      mbar_init(su32(&bars->xfull[b]), 1);
      mbar_init(su32(&bars->xempty[b]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(su32(&bars->tfull[b]), 1);
      mbar_init(su32(&bars->tempty[b]), kma::NEPI);
    }
    mbar_init(su32(&bars->ohfull), kma::NFIN);
    mbar_init(su32(&bars->ohempty), 1);
    mbar_init(su32(&bars->sumdone), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(su32(&bars->xready[b]), kma::NEPI);
      mbar_init(su32(&bars->xfree[b]), kma::NFIN);
    }
    mbar_init(su32(&bars->epidone), kma::NFIN);
    fence_barrier_init();
  }
  if (warp == kma::MMA_WARP) {
    tc_alloc(su32(&sMisc[0]), 512);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];
  const uint32_t tSum = tmem + 256;
  const uint32_t IDS = idesc_bf16(128, GP, false);
  constexpr uint32_t IDA = idesc_bf16_mn(128, D, true, true);
  // error bound of one score: 2 |x.w_hi + x.w_lo - x.w| <= 2 (2^-18 + 2 D 2^-24) ||x|| ||w||
  const float kc = 2.f * (3.814697265625e-06f + 2.f * D * 5.9604644775390625e-08f);
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  int it = 0, sg = 0;   // running tile / segment counters (identical across roles)
  bool ok = true;
  int prev_c[2] = {-1, -1};   // finisher: chunk of each of its rows' one in the one-hot tile
  // the one-hot tile starts all zero (the finisher then only moves each row's one)
  for (int e = tid; e < (int)(kOH / 16); e += kma::NT)
    *reinterpret_cast<uint4*>(smem + XS * kX + 16 * e) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();
  for (int s0 = t0; s0 < t1 && ok;) {
    const int bh = s0 / T;
    const int s1 = min(t1, (bh + 1) * T);
    const int slot = blockIdx.x * maxh + (bh - t0 / T);
    const size_t head = (size_t)bh * N;
    // ---- this head's weights (every role is idle here)
    __syncthreads();
    for (int e = tid; e < GP * CPR; e += kma::NT) {
      const int r = e / CPR, c = e - r * CPR;
      const size_t off = ((size_t)bh * GP + r) * D + c * 8;
      cp_async16(sWh + tile_off(r, c, GP), w_hi + off, true);
      cp_async16(sWl + tile_off(r, c, GP), w_lo + off, true);
    }
    float wm = 0.f;
    for (int g = tid; g < GP; g += kma::NT) {
      sBias[g] = bias[(size_t)bh * GP + g];
      sCnt[g] = 0;
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

    if (warp == kma::LOAD_WARP) {
      // ---------------- loads (rows past this head's N belong to the next head or read as
      // zeros; their labels and one-hot rows are never used) ----------------
      if (lane == 0) {
        for (int i = s0; i < s1 && ok; ++i, ++it) {
          const int xb = it % XS, n0 = (i - bh * T) * 128;
          if (it >= XS) ok = wait(bars->xempty[xb], ((it / XS) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(su32(&bars->xfull[xb]), kX);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_2d(sX + xb * kX + h * 16384, &tmx, 64 * h, (int)(head + n0), su32(&bars->xfull[xb]));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      it = __shfl_sync(0xffffffffu, it, 0);
    } else if (warp == kma::MMA_WARP) {
      // ---------------- MMA ----------------
      // Scores and sums are issued as their inputs become ready, not in a fixed order: the
      // scores of a later tile (needing its X tile and a free score buffer) do not wait
      // behind the sums of an earlier tile (needing that tile's one-hot rows).
      if (lane == 0) {
        const int first = it, last = it + (s1 - s0);
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
          if (nm < ns && mbar_test(su32(&bars->ohfull), nm & 1)) {
            const int xj = nm % XS;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              tc_mma(tSum, sdesc(sOH + k * 2048, 16384, 1024), sdesc(sX + xj * kX + k * 2048, 16384, 1024), IDA,
                     (nm > first || k > 0) ? 1u : 0u);
            tc_commit(su32(&bars->xempty[xj]));
            tc_commit(su32(&bars->ohempty));
            ++nm;
            moved = true;
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
        it = nm;
        tc_commit(su32(&bars->sumdone));
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      it = __shfl_sync(0xffffffffu, it, 0);
    } else if (warp >= kma::FIN_WARP) {
      // ---------------- finisher (warps 16-17): merge the quarters of rows f and f + 64,
      // labels, counts, flags, one-hot rows ----------------
      const int f = tid - kma::FIN_WARP * 32;
      for (int i = s0; i < s1 && ok; ++i, ++it) {
        const int b = it & 1;
        ok = __all_sync(0xffffffffu, wait(bars->xready[b], (it >> 1) & 1));
        if (!ok) break;
        int bi2[2];
        float best2[2], second2[2], xsum2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int r = f + 64 * u;
          // merge in column order, so a lower quarter wins ties
          kma::Half m = xchg[(b * kma::NQ + 0) * 128 + r];
          float xsum = m.xx;
#pragma unroll
          for (int q = 1; q < kma::NQ; ++q) {
            const kma::Half o = xchg[(b * kma::NQ + q) * 128 + r];
            xsum += o.xx;
            const bool take = o.best < m.best;
            m.second = take ? fminf(m.best, o.second) : fminf(m.second, o.best);
            if (take) { m.best = o.best; m.bi = o.bi; }
          }
          bi2[u] = m.bi;
          best2[u] = m.best;
          second2[u] = m.second;
          xsum2[u] = xsum;
        }
        // xchg[b] may take tile it + 2
        mbar_arrive(su32(&bars->xfree[b]));
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int r = f + 64 * u, row = (i - bh * T) * 128 + r;
          if (row < N) {
            const float best = best2[u], second = second2[u];
            const int bi = bi2[u];
            const float bound = kc * sqrtf(xsum2[u]) * wmax + 1e-6f * (fabsf(best) + fabsf(second));
            labels[head + row] = bi;
            atomicAdd(&sCnt[bi], 1);
            if (second - best > 2.f * bound) {
              if (trace) trace[head + row] = bi;
            } else {
              const int fs = atomicAdd(&flag_count[bh], 1);
              flag_rows[head + fs] = row;
            }
          }
        }
        // one-hot rows of this tile, once the previous sums read theirs: the tile holds the
        // previous tile's ones (all zero at the start), so a row clears the 16-byte chunk of
        // its previous one and sets the chunk of its new one (rows past N stay zero)
        if (it >= 1) ok = __all_sync(0xffffffffu, wait(bars->ohempty, (it - 1) & 1));
        if (!ok) break;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int r = f + 64 * u;
          const bool in = (i - bh * T) * 128 + r < N;
          const int bi = bi2[u];
          const int c_new = in ? (bi >> 3) : -1;
          if (prev_c[u] >= 0 && prev_c[u] != c_new)
            *reinterpret_cast<uint4*>(smem + XS * kX + tile_off(r, prev_c[u], 128)) = make_uint4(0u, 0u, 0u, 0u);
          if (c_new >= 0) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            const uint32_t one = 0x3F80u << (16 * (bi & 1));   // bf16 1.0 in the low or high half
            const int wd = (bi & 7) >> 1;
            if (wd == 0) v.x = one; else if (wd == 1) v.y = one; else if (wd == 2) v.z = one; else v.w = one;
            *reinterpret_cast<uint4*>(smem + XS * kX + tile_off(r, c_new, 128)) = v;
          }
          prev_c[u] = c_new;
        }
        fence_proxy_async();
        mbar_arrive(su32(&bars->ohfull));
      }
      // every row's count of this head is in sCnt
      mbar_arrive(su32(&bars->epidone));
    } else {
      // ---------------- argmin per column quarter (warps 0-15) ----------------
      const int hf = warp >> 2;                 // column quarter
      const int r = (warp & 3) * 32 + lane;     // row = TMEM lane
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      for (int i = s0; i < s1 && ok; ++i, ++it) {
        const int b = it & 1, xb = it % XS;
        // scores ready; the X tile (read below for ||x||) completed before them
        ok = __all_sync(0xffffffffu, wait(bars->tfull[b], (it >> 1) & 1) && wait(bars->xfull[xb], (it / XS) & 1));
        if (!ok) break;
        tc_fence_after();
        // argmin and runner-up of bias_g - 2 s_g over this quarter, in four interleaved sets
        float bst[4], snd[4];
        int bix[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) { bst[q] = __int_as_float(0x7f800000); snd[q] = bst[q]; bix[q] = 0; }
        {
          const int cb = hf * 32;
          if (cb < GP) {
            uint32_t v[32];
            tc_ld32(tmem + 128 * b + lane_off + cb, v);
            const uint64_t m2 = f2pack(-2.f, -2.f);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float sc2[2];
              f2unpack(ffma2(m2, f2pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                             f2pack(sBias[cb + e], sBias[cb + e + 1])), sc2[0], sc2[1]);
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int q = (e + u) & 3;
                const float sc = sc2[u];
                snd[q] = fminf(snd[q], fmaxf(bst[q], sc));
                bix[q] = sc < bst[q] ? cb + e + u : bix[q];
                bst[q] = fminf(bst[q], sc);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(su32(&bars->tempty[b]));
        kma::Half h;
        h.best = bst[0]; h.second = snd[0]; h.bi = bix[0];
#pragma unroll
        for (int q = 1; q < 4; ++q) {
          const bool take = bst[q] < h.best || (bst[q] == h.best && bix[q] < h.bi);
          h.second = take ? fminf(h.best, snd[q]) : fminf(h.second, bst[q]);
          if (take) { h.best = bst[q]; h.bi = bix[q]; }
        }
        // ||x||^2 of this quarter of the row, from the swizzled tile
        float xx = 0.f;
#pragma unroll
        for (int c = 0; c < CPR / kma::NQ; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(smem + xb * kX + tile_off(r, hf * (CPR / kma::NQ) + c, 128));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 fl = __bfloat1622float2(h2[e]);
            xx = fmaf(fl.x, fl.x, fmaf(fl.y, fl.y, xx));
          }
        }
        h.xx = xx;
        // the finisher has read xchg[b] of tile it - 2
        if (it >= 2) ok = __all_sync(0xffffffffu, wait(bars->xfree[b], ((it >> 1) - 1) & 1));
        if (!ok) break;
        xchg[(b * kma::NQ + hf) * 128 + r] = h;
        mbar_arrive(su32(&bars->xready[b]));
      }
      // ---- sums and counts of this head -> partial slot (each quarter writes 32 columns)
      if (ok) ok = __all_sync(0xffffffffu, wait(bars->sumdone, sg & 1));
      if (ok) ok = __all_sync(0xffffffffu, wait(bars->epidone, sg & 1));
      if (ok) {
        tc_fence_after();
        for (int cb = hf * 32; cb < D; cb += 32 * kma::NQ) {
          uint32_t v[32];
          tc_ld32(tSum + lane_off + cb, v);
          if (r < GP) {
            float* dst = psum + ((size_t)slot * GP + r) * D + cb;
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                                __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
          }
        }
        if (r < GP && hf == 0) pcnt[(size_t)slot * GP + r] = sCnt[r];
        tc_fence_before();
      }
    }
    ++sg;
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    s0 = s1;
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
                                                       const int* __restrict__ flag_count,
                                                       const int* __restrict__ flag_rows, int* __restrict__ labels,
                                                       int* __restrict__ trace, int* __restrict__ corr_count,
                                                       int4* __restrict__ corr) {
  extern __shared__ __align__(16) float sr[];
  const int bh = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int cnt = flag_count[bh];
  if ((int)blockIdx.x * 16 >= cnt) return;
  float* sA = sr;                       // [D][d + 1]
  float* sNu = sA + D * (d + 1);        // [G][DT + 1]
  float* sx = sNu + G * (DT + 1);       // [16][d]
  float* sy = sx + 16 * d;              // [16][DT]
  const size_t head = (size_t)bh * N;
  const float* Ah = A + a_head * bh;
  const float* nuh = nu + (size_t)bh * G * DT;
  // staging loops unrolled so that each thread keeps several loads in flight
#pragma unroll 8
  for (int e = threadIdx.x; e < D * d; e += 512) {
    const int j = e / d, c = e - j * d;
    sA[j * (d + 1) + c] = Ah[(size_t)j * sj + (size_t)c * sc];
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
    const int row = flag_rows[head + i];
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
          if (tile >= 2) ok = __all_sync(0xffffffffu, wait(bars->xempty[b], ((tile >> 1) - 1) & 1));
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int r = 32 * k + lane;
            int myrow = -1;
            if (r < nr) {
              myrow = perm_q[head + t0 + r];
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
  return (size_t)km::kma::XS * 128 * D * 2 + (size_t)128 * 128 * 2 + 2 * (size_t)GP * D * 2 +
         2 * km::kma::NQ * 128 * sizeof(km::kma::Half) + (size_t)GP * 8 + sizeof(km::kma::Bars) + 16;
}

KmPlan kmeans_plan(int BH, int N) {
  KmPlan pl{};
  pl.T = ceil_div(N, 128);
  pl.total = BH * pl.T;
  pl.grid = pl.total < kKmeansCtas ? pl.total : kKmeansCtas;
  pl.per = ceil_div(pl.total, pl.grid);
  pl.maxh = pl.per / pl.T + 2;
  return pl;
}

cudaError_t launch_seed_rows(const void* X, int BH, int N, int d, int G, uint64_t seed, HeadMap hm, int purpose,
                             float* m, int* init_out, int* err, cudaStream_t st) {
  const size_t sm = (size_t)2 * G * 4;
  cudaFuncSetAttribute(km::k_seed_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_seed_rows<<<BH, 256, sm, st>>>((const __nv_bfloat16*)X, N, d, G, seed, hm, purpose, m, init_out, err);
  return cudaGetLastError();
}

size_t centroid_weights_smem(int d, int D) {
  return (size_t)km::WG_PER_CTA * d * 8 + km::WG_PER_CTA * 4 +
         ((size_t)D * (d + 1) + (size_t)km::WG_PER_CTA * d + (size_t)km::WG_PER_CTA * 128) * 4;
}

cudaError_t launch_centroid_weights(float* m, int BH, int G, int d, const float* A, size_t a_head, int sj, int sc,
                                    float a_scale, int D, int DT, int mode, const float* psum, const int* pcnt,
                                    const int* corr_count, const void* corr, const void* X, int N, float* nu,
                                    float* bias, float* wnorm, void* w_hi, void* w_lo, int* err, cudaStream_t st) {
  const int GP = kmeans_gp(G);
  const size_t sm = centroid_weights_smem(d, D);
  const KmPlan pl = kmeans_plan(BH, N);
  km::KmPartials pp{psum, pcnt, corr_count, (const int4*)corr, (const __nv_bfloat16*)X, N, pl.T, pl.per, pl.maxh,
                    pl.grid};
  cudaFuncSetAttribute(km::k_centroid_weights, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_centroid_weights<<<dim3(ceil_div(GP, km::WG_PER_CTA), BH), km::CW_THREADS, sm, st>>>(
      m, G, GP, d, A, a_head, sj, sc, a_scale, D, DT, mode, pp, nu, bias, wnorm, (__nv_bfloat16*)w_hi,
      (__nv_bfloat16*)w_lo, err);
  return cudaGetLastError();
}

cudaError_t launch_assign_acc(const void* X, int BH, int N, int d, int G, const void* w_hi, const void* w_lo,
                              const float* bias, const float* wnorm, int* labels, int* trace, int* flag_count,
                              int* flag_rows, float* psum, int* pcnt, int* err, cudaStream_t st) {
  const int GP = kmeans_gp(G);
  const size_t sm = assign_acc_smem(d, GP);
  const KmPlan pl = kmeans_plan(BH, N);
  CUtensorMap tmx;
  cudaError_t e = make_tmap_bf16_rows(&tmx, X, (unsigned long long)BH * N, d, 128);
  if (e != cudaSuccess) return e;
  if (d == 64) {
    cudaFuncSetAttribute(km::k_assign_acc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_assign_acc<64><<<pl.grid, km::kma::NT, sm, st>>>(
        tmx, N, GP, pl.T, pl.total, pl.per, pl.maxh, (const __nv_bfloat16*)w_hi, (const __nv_bfloat16*)w_lo, bias,
        wnorm, labels, trace, flag_count, flag_rows, psum, pcnt, err);
  } else {
    cudaFuncSetAttribute(km::k_assign_acc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_assign_acc<128><<<pl.grid, km::kma::NT, sm, st>>>(
        tmx, N, GP, pl.T, pl.total, pl.per, pl.maxh, (const __nv_bfloat16*)w_hi, (const __nv_bfloat16*)w_lo, bias,
        wnorm, labels, trace, flag_count, flag_rows, psum, pcnt, err);
  }
  return cudaGetLastError();
}

size_t recheck_smem(int d, int D, int DT, int G) {
  return ((size_t)D * (d + 1) + (size_t)G * (DT + 1) + 16 * (size_t)d + 16 * (size_t)DT) * 4;
}

template <int DT>
static cudaError_t recheck_dt(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                              float a_scale, int D, const float* nu, int G, const int* flag_count,
                              const int* flag_rows, int* labels, int* trace, int* corr_count, void* corr,
                              cudaStream_t st) {
  const size_t sm = recheck_smem(d, D, DT, G);
  cudaFuncSetAttribute(km::k_assign_recheck<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_assign_recheck<DT><<<dim3(km::RC_PER_HEAD, BH), 512, sm, st>>>((const __nv_bfloat16*)X, N, d, A, a_head, sj,
                                                                      sc, a_scale, D, nu, G, flag_count, flag_rows,
                                                                      labels, trace, corr_count, (int4*)corr);
  return cudaGetLastError();
}

cudaError_t launch_assign_recheck(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                                  float a_scale, int D, const float* nu, int G, const int* flag_count,
                                  const int* flag_rows, int* labels, int* trace, int* corr_count, void* corr,
                                  cudaStream_t st) {
  switch (kmeans_dt(D)) {
    case 8: return recheck_dt<8>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, corr_count, corr, st);
    case 16: return recheck_dt<16>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, corr_count, corr, st);
    case 32: return recheck_dt<32>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, corr_count, corr, st);
    case 64: return recheck_dt<64>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, corr_count, corr, st);
    case 128: return recheck_dt<128>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, corr_count, corr, st);
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
