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
                                                  uint64_t seed, int purpose, float* __restrict__ m,
                                                  int* __restrict__ init_out, int* err) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* mkey = reinterpret_cast<int*>(smem);
  int* mval = mkey + kMapCap;
  int* sidx = mval + kMapCap;
  const int bh = blockIdx.x, tid = threadIdx.x;
  SlotMap map{mkey, mval, kMapCap};
  map.clear_all(tid, blockDim.x);
  __syncthreads();
  if (tid == 0) {
    SplitMix64 g(stream_state(seed, bh, purpose));
    if (!draw_without_replacement(g, N, G, map, sidx)) set_error(err, DERR_DRAW);
  }
  __syncthreads();
  for (int e = tid; e < G * d; e += blockDim.x) {
    const int g = e / d, c = e - g * d;
    m[(size_t)bh * G * d + e] = bf2f(X[((size_t)bh * N + sidx[g]) * d + c]);
  }
  if (init_out)
    for (int g = tid; g < G; g += blockDim.x) init_out[(size_t)bh * G + g] = sidx[g];
}

// ---------------------------------------------------------------------------
// Centroid weights.  A(j, c) = a_scale * A[j * sj + c * sc] (D x d) is staged once per
// CTA in shared memory as sA[j][c] with row stride d + 1 (conflict-free both ways).
//   nu = A m (fp32, sequential over c), bias = ||nu||^2 (sequential over j),
//   w = A^T nu -> w_hi = bf16(w), w_lo = bf16(w - w_hi); wnorm = ||w||.
// Rows g in [G, GP) are padding: w = 0, bias = +inf.
// grid = (ceil(GP / WG_PER_CTA), BH), block = 128.
// ---------------------------------------------------------------------------
constexpr int WG_PER_CTA = 16;

__global__ void __launch_bounds__(128) k_centroid_weights(const float* __restrict__ m, int G, int GP, int d,
                                                         const float* __restrict__ A, size_t a_head, int sj,
                                                         int sc, float a_scale, int D, int DT,
                                                         float* __restrict__ nu, float* __restrict__ bias,
                                                         float* __restrict__ wnorm,
                                                         __nv_bfloat16* __restrict__ w_hi,
                                                         __nv_bfloat16* __restrict__ w_lo) {
  extern __shared__ __align__(16) float sw[];
  float* sA = sw;                        // [D][d + 1]
  float* sm_m = sA + D * (d + 1);        // [d]
  float* sm_nu = sm_m + d;               // [128]
  float* sm_w = sm_nu + 128;             // [d]
  const int bh = blockIdx.y, tid = threadIdx.x;
  const float* Ah = A + a_head * bh;
  for (int e = tid; e < D * d; e += 128) {
    const int j = e / d, c = e - j * d;
    sA[j * (d + 1) + c] = Ah[(size_t)j * sj + (size_t)c * sc];
  }
  __syncthreads();
  const int g0 = blockIdx.x * WG_PER_CTA, g1 = min(GP, g0 + WG_PER_CTA);
  for (int g = g0; g < g1; ++g) {
    const size_t wrow = ((size_t)bh * GP + g) * d;
    if (g >= G) {
      for (int c = tid; c < d; c += 128) {
        w_hi[wrow + c] = __float2bfloat16(0.f);
        w_lo[wrow + c] = __float2bfloat16(0.f);
      }
      if (tid == 0) {
        bias[(size_t)bh * GP + g] = __int_as_float(0x7f800000);
        wnorm[(size_t)bh * GP + g] = 0.f;
      }
      continue;
    }
    for (int c = tid; c < d; c += 128) sm_m[c] = m[((size_t)bh * G + g) * d + c];
    __syncthreads();
    for (int j = tid; j < D; j += 128) {
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(sA[j * (d + 1) + c], sm_m[c], acc);
      sm_nu[j] = a_scale * acc;
    }
    __syncthreads();
    for (int j = tid; j < DT; j += 128) nu[((size_t)bh * G + g) * DT + j] = j < D ? sm_nu[j] : 0.f;
    for (int c = tid; c < d; c += 128) {
      float acc = 0.f;
      for (int j = 0; j < D; ++j) acc = fmaf(sA[j * (d + 1) + c], sm_nu[j], acc);
      const float w = a_scale * acc;
      sm_w[c] = w;
      const __nv_bfloat16 hi = __float2bfloat16(w);
      w_hi[wrow + c] = hi;
      w_lo[wrow + c] = __float2bfloat16(w - __bfloat162float(hi));
    }
    __syncthreads();
    if (tid == 0) {
      float b = 0.f, n2 = 0.f;
      for (int j = 0; j < D; ++j) b = fmaf(sm_nu[j], sm_nu[j], b);
      for (int c = 0; c < d; ++c) n2 = fmaf(sm_w[c], sm_w[c], n2);
      bias[(size_t)bh * GP + g] = b;
      wnorm[(size_t)bh * GP + g] = sqrtf(n2);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Tensor-core assignment.  One CTA = TPC consecutive 128-row tiles of one head.
// 128 threads: every thread owns one row in the epilogue (TMEM lane = row); thread 0
// issues the MMAs; warp 0 owns the TMEM allocation (128 columns).
// ---------------------------------------------------------------------------
constexpr int TPC = 4;

template <int D>
__global__ void __launch_bounds__(128) k_assign_tc(const __nv_bfloat16* __restrict__ X, int N, int GP,
                                                  const __nv_bfloat16* __restrict__ w_hi,
                                                  const __nv_bfloat16* __restrict__ w_lo,
                                                  const float* __restrict__ bias, const float* __restrict__ wnorm,
                                                  int* __restrict__ labels, int* __restrict__ trace,
                                                  int* __restrict__ flag_count, int* __restrict__ flag_rows,
                                                  int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = su32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - raw);
  constexpr uint32_t kX = 128u * D * 2u;          // X tile bytes
  const uint32_t kW = (uint32_t)GP * D * 2u;      // one W tile
  const uint32_t sX = base, sWh = base + kX, sWl = sWh + kW;
  float* sBias = reinterpret_cast<float*>(smem + kX + 2 * kW);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sBias + 128);
  int* sMisc = reinterpret_cast<int*>(bar + 1);  // [0] tmem, [1] abort, [2] wmax bits
  volatile int* abort_flag = sMisc + 1;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y;
  const size_t head = (size_t)bh * N;
  constexpr int CPR = D / 8;

  // weights, bias, max ||w||
  for (int e = tid; e < GP * CPR; e += 128) {
    const int r = e / CPR, c = e - r * CPR;
    const size_t off = ((size_t)bh * GP + r) * D + c * 8;
    cp_async16(sWh + tile_off(r, c, GP), w_hi + off, true);
    cp_async16(sWl + tile_off(r, c, GP), w_lo + off, true);
  }
  float wmax = 0.f;
  for (int g = tid; g < GP; g += 128) {
    sBias[g] = bias[(size_t)bh * GP + g];
    wmax = fmaxf(wmax, wnorm[(size_t)bh * GP + g]);
  }
  wmax = warp_max(wmax);
  if (tid == 0) {
    sMisc[1] = 0;
    sMisc[2] = 0;
    mbar_init(su32(bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if ((tid & 31) == 0) atomicMax(&sMisc[2], __float_as_int(wmax));  // non-negative floats order as ints
  if (warp == 0) {
    tc_alloc(su32(&sMisc[0]), 128);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];
  wmax = __int_as_float(sMisc[2]);
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(GP >> 3) << 17) | (8u << 24);
  // error bound of one score: 2 |x.w_hi + x.w_lo - x.w| <= 2 (2^-18 + 2 D 2^-24) ||x|| ||w||
  const float kc = 2.f * (3.814697265625e-06f + 2.f * D * 5.9604644775390625e-08f);

  for (int it = 0; it < TPC; ++it) {
    const int n0 = (blockIdx.x * TPC + it) * 128;
    if (n0 >= N) break;
    for (int e = tid; e < 128 * CPR; e += 128) {
      const int r = e / CPR, c = e - r * CPR;
      const bool ok = n0 + r < N;
      cp_async16(sX + tile_off(r, c, 128), X + (head + (ok ? n0 + r : 0)) * D + c * 8, ok);
    }
    cp_async_wait_all();
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
        const uint32_t ow = (k >> 2) * (GP * 128) + (k & 3) * 32;
        tc_mma(tmem, sdesc(sX + ox, 16, 1024), sdesc(sWh + ow, 16, 1024), idesc, k > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
        const uint32_t ow = (k >> 2) * (GP * 128) + (k & 3) * 32;
        tc_mma(tmem, sdesc(sX + ox, 16, 1024), sdesc(sWl + ow, 16, 1024), idesc, 1u);
      }
      tc_commit(su32(bar));
    }
    // ||x|| of this thread's row (from the swizzled tile)
    float xx = 0.f;
#pragma unroll
    for (int c = 0; c < CPR; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(smem + tile_off(tid, c, 128));
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        xx = fmaf(f.x, f.x, fmaf(f.y, f.y, xx));
      }
    }
    // CTA-uniform outcome, so every thread takes the same barriers afterwards
    const bool ok = __syncthreads_and(bounded_wait(su32(bar), it & 1, abort_flag, err) ? 1 : 0) != 0;
    if (!ok) break;
    tc_fence_after();
    float best = __int_as_float(0x7f800000), second = best;
    int bi = 0;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < GP; c0 += 32) {
      uint32_t r[32];
      tc_ld32(tmem + lane_off + c0, r);
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float v = sBias[c0 + e] - 2.f * __uint_as_float(r[e]);
        if (v < best) { second = best; best = v; bi = c0 + e; }
        else if (v < second) second = v;
      }
    }
    const int row = n0 + tid;
    if (row < N) {
      const float bound = kc * sqrtf(xx) * wmax + 1e-6f * (fabsf(best) + fabsf(second));
      if (second - best > 2.f * bound) {
        labels[head + row] = bi;
        if (trace) trace[head + row] = bi;
      } else {
        const int slot = atomicAdd(&flag_count[bh], 1);
        flag_rows[head + slot] = row;
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tc_dealloc(tmem, 128);
}

// ---------------------------------------------------------------------------
// Exact re-assignment of the uncertified rows: y = A x (fp32, sequential over c),
// dist_g = sum_c (y_c - nu_gc)^2 (sequential fp32 fma over c), argmin with ties to the
// lowest g.  A and the centroids are staged in shared memory (padded rows); one warp per
// row.  grid = (RC_PER_HEAD, BH), block = 512.
// ---------------------------------------------------------------------------
constexpr int RC_PER_HEAD = 8;

template <int DT>
__global__ void __launch_bounds__(512) k_assign_recheck(const __nv_bfloat16* __restrict__ X, int N, int d,
                                                       const float* __restrict__ A, size_t a_head, int sj, int sc,
                                                       float a_scale, int D, const float* __restrict__ nu, int G,
                                                       const int* __restrict__ flag_count,
                                                       const int* __restrict__ flag_rows, int* __restrict__ labels,
                                                       int* __restrict__ trace) {
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
  for (int e = threadIdx.x; e < D * d; e += 512) {
    const int j = e / d, c = e - j * d;
    sA[j * (d + 1) + c] = Ah[(size_t)j * sj + (size_t)c * sc];
  }
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
      labels[head + row] = bi;
      if (trace) trace[head + row] = bi;
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Segment means of raw rows: m[g] = mean over permuted positions of group g of X[perm]
// (fp64 sums; warp w sums members w, w+8, ...; warps combined in order).  Empty groups
// keep m.  grid = (G, BH), block = 256.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_segment_mean_rows(const __nv_bfloat16* __restrict__ X, int N, int G,
                                                          const int* __restrict__ perm,
                                                          const int* __restrict__ offsets, float* __restrict__ m) {
  constexpr int PL = D / 32;  // columns per lane
  __shared__ double part[8][D];
  const int g = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int s0 = offsets[(size_t)bh * (G + 1) + g], s1 = offsets[(size_t)bh * (G + 1) + g + 1];
  if (s1 == s0) return;
  const int* pm = perm + (size_t)bh * N;
  const __nv_bfloat16* Xh = X + (size_t)bh * N * D;
  double acc[PL];
#pragma unroll
  for (int e = 0; e < PL; ++e) acc[e] = 0.0;
  for (int s = s0 + warp; s < s1; s += 8) {
    const __nv_bfloat16* row = Xh + (size_t)pm[s] * D + lane * PL;
    if constexpr (PL == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(row);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
      const float2 a = __bfloat1622float2(h2[0]), b = __bfloat1622float2(h2[1]);
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += b.x;
      acc[3] += b.y;
    } else {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(row));
      acc[0] += a.x;
      acc[1] += a.y;
    }
  }
#pragma unroll
  for (int e = 0; e < PL; ++e) part[warp][lane * PL + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += part[w][c];
    m[((size_t)bh * G + g) * D + c] = (float)(t / (double)(s1 - s0));
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

// Roles of the 192 threads of the persistent cell-mass kernel: warps 0-3 take the softmax
// of tile row r = TMEM lane r and the column sums, warp 4 allocates TMEM and its lane 0
// issues the MMAs, warp 5 gathers the tile's query rows through perm_q (cp.async) into a
// two-deep ring.  CTA b takes the (head, query group) items [b per, (b+1) per) in order;
// the K/V centroid parts of a head are reloaded when the head changes.
namespace cmk {
constexpr int NT = 192;
constexpr int MMA_WARP = 4;
constexpr int LOAD_WARP = 5;
struct Bars {
  uint64_t xfull[2], xempty[2], tfull[2], tempty[2];
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
  float* part = reinterpret_cast<float*>(smem + 2 * kX + 3 * kC);   // [4][GP]
  float* colacc = part + 4 * GP;                                     // [GP]
  float* lnn = colacc + GP;                                          // [GP] log2 n_g or -inf
  cmk::Bars* bars = reinterpret_cast<cmk::Bars*>(lnn + GP);
  int* sMisc = reinterpret_cast<int*>(bars + 1);                     // [0] tmem, [1] abort
  volatile int* abort_flag = sMisc + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float NEG_INF = __int_as_float(0xff800000);

  if (tid == 0) {
    sMisc[1] = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(su32(&bars->xfull[b]), 32);
      mbar_init(su32(&bars->xempty[b]), 1);
      mbar_init(su32(&bars->tfull[b]), 1);
      mbar_init(su32(&bars->tempty[b]), 128);
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
    } else if (warp < 4) {
      // ---------------- softmax + column sums ----------------
      const int r = tid;   // tile row = TMEM lane
      const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
      for (int a = a0; a < a1 && ok; ++a) {
        const int n_a = qo[a + 1] - qo[a];
        if (n_a == 0) {
          if (r < Gk) mass[((size_t)bh * Gq + a) * Gk + r] = 0.f;
          continue;
        }
        for (int t0 = qo[a]; t0 < qo[a + 1]; t0 += 128, ++tile) {
          const int b = tile & 1, nr = min(128, qo[a + 1] - t0);
          ok = __all_sync(0xffffffffu, wait(bars->tfull[b], (tile >> 1) & 1));
          if (!ok) break;
          tc_fence_after();
          float v[128];
#pragma unroll
          for (int c0 = 0; c0 < 128; c0 += 32) {
            if (c0 < GP) {
              uint32_t u[32];
              tc_ld32(tmem + 128 * b + lane_off + c0, u);
#pragma unroll
              for (int e = 0; e < 32; ++e) v[c0 + e] = __uint_as_float(u[e]);
            }
          }
          tc_fence_before();
          mbar_arrive(su32(&bars->tempty[b]));
          float mx = NEG_INF;
#pragma unroll
          for (int g = 0; g < 128; ++g) {
            if (g < GP) {
              const float ln = lnn[g];
              v[g] = ln == NEG_INF ? NEG_INF : fmaf(v[g], scale_log2, ln);
              mx = fmaxf(mx, v[g]);
            }
          }
          float sum = 0.f;
#pragma unroll
          for (int g = 0; g < 128; ++g) {
            if (g < GP) {
              v[g] = v[g] == NEG_INF ? 0.f : ex2(v[g] - mx);
              sum += v[g];
            }
          }
          const float inv = (r < nr && sum > 0.f) ? 1.f / sum : 0.f;
#pragma unroll
          for (int c0 = 0; c0 < 128; c0 += 32) {
            if (c0 < GP) {
              float w[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) w[e] = v[c0 + e] * inv;
              part[warp * GP + c0 + lane] = lane_column_sum32(w, lane);
            }
          }
          named_sync(1, 128);
          if (r < GP) {
            colacc[r] += (part[r] + part[GP + r]) + (part[2 * GP + r] + part[3 * GP + r]);
            if (t0 + 128 >= qo[a + 1]) {
              if (r < Gk) mass[((size_t)bh * Gq + a) * Gk + r] = colacc[r] / (float)n_a;
              colacc[r] = 0.f;
            }
          }
          named_sync(1, 128);
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

size_t assign_tc_smem(int D, int GP) {
  return 1024 + (size_t)128 * D * 2 + 2 * (size_t)GP * D * 2 + 128 * 4 + 8 + 16;
}

cudaError_t launch_seed_rows(const void* X, int BH, int N, int d, int G, uint64_t seed, int purpose, float* m,
                             int* init_out, int* err, cudaStream_t st) {
  const size_t sm = (size_t)(2 * km::kMapCap + G) * 4;
  cudaFuncSetAttribute(km::k_seed_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_seed_rows<<<BH, 256, sm, st>>>((const __nv_bfloat16*)X, N, d, G, seed, purpose, m, init_out, err);
  return cudaGetLastError();
}

size_t centroid_weights_smem(int d, int D) { return ((size_t)D * (d + 1) + 2 * d + 128) * 4; }

cudaError_t launch_centroid_weights(const float* m, int BH, int G, int d, const float* A, size_t a_head, int sj,
                                    int sc, float a_scale, int D, int DT, float* nu, float* bias, float* wnorm,
                                    void* w_hi, void* w_lo, cudaStream_t st) {
  const int GP = kmeans_gp(G);
  const size_t sm = centroid_weights_smem(d, D);
  cudaFuncSetAttribute(km::k_centroid_weights, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_centroid_weights<<<dim3(ceil_div(GP, km::WG_PER_CTA), BH), 128, sm, st>>>(
      m, G, GP, d, A, a_head, sj, sc, a_scale, D, DT, nu, bias, wnorm, (__nv_bfloat16*)w_hi, (__nv_bfloat16*)w_lo);
  return cudaGetLastError();
}

cudaError_t launch_assign_tc(const void* X, int BH, int N, int d, int G, const void* w_hi, const void* w_lo,
                             const float* bias, const float* wnorm, int* labels, int* trace, int* flag_count,
                             int* flag_rows, int* err, cudaStream_t st) {
  const int GP = kmeans_gp(G);
  const size_t sm = assign_tc_smem(d, GP);
  dim3 grid(ceil_div(N, 128 * km::TPC), BH);
  if (d == 64) {
    cudaFuncSetAttribute(km::k_assign_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_assign_tc<64><<<grid, 128, sm, st>>>((const __nv_bfloat16*)X, N, GP, (const __nv_bfloat16*)w_hi,
                                               (const __nv_bfloat16*)w_lo, bias, wnorm, labels, trace, flag_count,
                                               flag_rows, err);
  } else {
    cudaFuncSetAttribute(km::k_assign_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_assign_tc<128><<<grid, 128, sm, st>>>((const __nv_bfloat16*)X, N, GP, (const __nv_bfloat16*)w_hi,
                                                (const __nv_bfloat16*)w_lo, bias, wnorm, labels, trace, flag_count,
                                                flag_rows, err);
  }
  return cudaGetLastError();
}

size_t recheck_smem(int d, int D, int DT, int G) {
  return ((size_t)D * (d + 1) + (size_t)G * (DT + 1) + 16 * (size_t)d + 16 * (size_t)DT) * 4;
}

template <int DT>
static cudaError_t recheck_dt(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                              float a_scale, int D, const float* nu, int G, const int* flag_count,
                              const int* flag_rows, int* labels, int* trace, cudaStream_t st) {
  const size_t sm = recheck_smem(d, D, DT, G);
  cudaFuncSetAttribute(km::k_assign_recheck<DT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  km::k_assign_recheck<DT><<<dim3(km::RC_PER_HEAD, BH), 512, sm, st>>>((const __nv_bfloat16*)X, N, d, A, a_head, sj,
                                                                      sc, a_scale, D, nu, G, flag_count, flag_rows,
                                                                      labels, trace);
  return cudaGetLastError();
}

cudaError_t launch_assign_recheck(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                                  float a_scale, int D, const float* nu, int G, const int* flag_count,
                                  const int* flag_rows, int* labels, int* trace, cudaStream_t st) {
  switch (kmeans_dt(D)) {
    case 8: return recheck_dt<8>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, st);
    case 16: return recheck_dt<16>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, st);
    case 32: return recheck_dt<32>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, st);
    case 64: return recheck_dt<64>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, st);
    case 128: return recheck_dt<128>(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, flag_count, flag_rows, labels, trace, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_segment_mean_rows(const void* X, int BH, int N, int d, int G, const int* perm, const int* offsets,
                                     float* m, cudaStream_t st) {
  if (d == 64)
    km::k_segment_mean_rows<64><<<dim3(G, BH), 256, 0, st>>>((const __nv_bfloat16*)X, N, G, perm, offsets, m);
  else
    km::k_segment_mean_rows<128><<<dim3(G, BH), 256, 0, st>>>((const __nv_bfloat16*)X, N, G, perm, offsets, m);
  return cudaGetLastError();
}

size_t cell_mass_tc_smem(int D, int GP) {
  return (size_t)2 * 128 * D * 2 + 3 * (size_t)GP * D * 2 + (size_t)6 * GP * 4 + sizeof(km::cmk::Bars) + 16;
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
                                float* mass, int* err, cudaStream_t st) {
  const int GP = kmeans_gp(Gk);
  km::k_split3<<<dim3(GP, BH), 128, 0, st>>>(C, Gk, GP, d, (__nv_bfloat16*)c1, (__nv_bfloat16*)c2,
                                            (__nv_bfloat16*)c3);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t sm = cell_mass_tc_smem(d, GP);
  const int nitems = BH * Gq;
  const int grid = nitems < sm_count() ? nitems : sm_count();
  const float scale_log2 = scale * 1.4426950408889634f;
  if (d == 64) {
    cudaFuncSetAttribute(km::k_cell_mass_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_cell_mass_tc<64><<<grid, km::cmk::NT, sm, st>>>((const __nv_bfloat16*)Q, N, Gq, Gk, GP, nitems, perm_q, qoff,
                                                         koff, (const __nv_bfloat16*)c1, (const __nv_bfloat16*)c2,
                                                         (const __nv_bfloat16*)c3, scale_log2, mass, err);
  } else {
    cudaFuncSetAttribute(km::k_cell_mass_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    km::k_cell_mass_tc<128><<<grid, km::cmk::NT, sm, st>>>((const __nv_bfloat16*)Q, N, Gq, Gk, GP, nitems, perm_q,
                                                          qoff, koff, (const __nv_bfloat16*)c1,
                                                          (const __nv_bfloat16*)c2, (const __nv_bfloat16*)c3,
                                                          scale_log2, mass, err);
  }
  return cudaGetLastError();
}

}  // namespace spr
