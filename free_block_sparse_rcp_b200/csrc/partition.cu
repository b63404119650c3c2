// Response-coupled partition kernels (gist.science technical summary, section 2.A;
// huashangw.com article, method walkthrough and sparse-execution section).
//
//   sample + metric   M_K = Q_s^T Q_s / M_s over M_s sampled query rows
//   eigen             leading r_e eigenpairs of M_K (single-CTA Jacobi)
//   key coordinates   y = Lambda^{1/2} U^T k (materialised for traces only)
//   (k-means itself: kmeans_tc.cu)
//   group sort        stable counting sort by label -> permutation + offsets
//   centroids         mean raw key of every K/V group
//   query coordinates z = s C q (materialised for traces only)
//   route             shared alpha by bisection under the pair budget
//   block mask        tile-level view of the route on the permuted layout
#include "common.cuh"
#include "symeig.cuh"
#include "kernels.h"

namespace spr {

// ---------------------------------------------------------------------------
// Sampled queries and M_K.  grid = BH, block = D * D / 16 (a 4 x 4 block of M_K per thread).
// ---------------------------------------------------------------------------
constexpr int kMapCap = 4096;

template <int D>
__global__ void __launch_bounds__(D * D / 16) k_sample_metric(const __nv_bfloat16* __restrict__ Q, int N,
                                                             int Ms, uint64_t seed, HeadMap hm,
                                                             float* __restrict__ metric,
                                                             int* __restrict__ sample_idx, int* err) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* sidx = reinterpret_cast<int*>(smem);                     // [Ms]
  float* qs = reinterpret_cast<float*>(sidx + ((Ms + 3) & ~3)); // [64][D]
  const int bh = blockIdx.x, tid = threadIdx.x;
  // the draw's offsets go to the (not yet used) row buffer: Ms <= kMapCap / 2 <= 64 D
  if (!draw_without_replacement_block(stream_state(seed, hm.global(bh), PURPOSE_QUERY_SAMPLE), N, Ms, kMapCap, sidx,
                                      reinterpret_cast<int*>(qs))) {
    if (tid == 0) set_error(err, DERR_DRAW);
    return;
  }
  for (int i = tid; i < Ms; i += blockDim.x) sample_idx[(size_t)bh * Ms + i] = sidx[i];
  // thread = a 4 x 4 block of M_K: rows 4 rb .. 4 rb + 3, columns 4 cb .. 4 cb + 3; every
  // entry is a sequential fp32 sum over the samples in draw order
  constexpr int CB = D / 4;
  const int rb = tid / CB, cb = tid - rb * CB;
  float acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) acc[j] = 0.f;
  const __nv_bfloat16* Qh = Q + (size_t)bh * N * D;
  for (int s0 = 0; s0 < Ms; s0 += 64) {
    const int ns = min(64, Ms - s0);
    for (int e = tid; e < ns * (D / 8); e += blockDim.x) {   // 16-byte pieces of the rows
      const int s = e / (D / 8), v = e - s * (D / 8);
      const uint4 x = *reinterpret_cast<const uint4*>(Qh + (size_t)sidx[s0 + s] * D + v * 8);
      const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
      const float2 f0 = __bfloat1622float2(x2[0]), f1 = __bfloat1622float2(x2[1]);
      const float2 f2 = __bfloat1622float2(x2[2]), f3 = __bfloat1622float2(x2[3]);
      float4* dst = reinterpret_cast<float4*>(qs + s * D + v * 8);
      dst[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
      dst[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
    }
    __syncthreads();
    for (int s = 0; s < ns; ++s) {
      const float4 qr = *reinterpret_cast<const float4*>(qs + s * D + 4 * rb);
      const float4 qc = *reinterpret_cast<const float4*>(qs + s * D + 4 * cb);
      const float vr[4] = {qr.x, qr.y, qr.z, qr.w}, vc[4] = {qc.x, qc.y, qc.z, qc.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a * 4 + b] = fmaf(vr[a], vc[b], acc[a * 4 + b]);
    }
    __syncthreads();
  }
  const float inv = 1.0f / (float)Ms;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const float4 v = make_float4(acc[a * 4] * inv, acc[a * 4 + 1] * inv, acc[a * 4 + 2] * inv, acc[a * 4 + 3] * inv);
    *reinterpret_cast<float4*>(metric + (size_t)bh * D * D + (size_t)(4 * rb + a) * D + 4 * cb) = v;
  }
}

// ---------------------------------------------------------------------------
// Leading eigenpairs of M_K (fp32 Householder + multisection + inverse iteration).
// grid = BH, block = 1024.  Writes eigval [BH, R] (clamped >= 0), eigvec [BH, D, R] and
// the projector P = U_R Lambda_R^{1/2} [BH, D, R].  lu: BH * 3 * D * R floats of scratch.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(1024) k_metric_eigen(const float* __restrict__ metric, int R,
                                                     float* __restrict__ eigval, float* __restrict__ eigvec,
                                                     float* __restrict__ proj, float* __restrict__ lu) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int LD = D + 1;
  const int ldz = R + 1;
  float* A = reinterpret_cast<float*>(smem);   // [D][D+1]
  float* Z = A + D * LD;                       // [D][R+1]
  float* lam = Z + D * ldz;                    // [64]
  float* sc = lam + 64;                        // SymEigScratch<float, D>
  const int bh = blockIdx.x;
#pragma unroll 8
  for (int i = threadIdx.x; i < D * D; i += blockDim.x) {
    const int r = i / D, c = i - r * D;
    A[r * LD + c] = metric[(size_t)bh * D * D + i];
  }
  __syncthreads();
  sym_top_eigen<float, D>(A, R, Z, ldz, lam, sc, lu + (size_t)bh * 3 * D * R);
  for (int e = threadIdx.x; e < D * R; e += blockDim.x) {
    const int c = e / R, k = e - c * R;
    const float l = fmaxf(lam[k], 0.f);
    const float u = Z[c * ldz + k];
    if (c == 0) eigval[(size_t)bh * R + k] = l;
    eigvec[(size_t)bh * D * R + e] = u;
    proj[(size_t)bh * D * R + e] = u * sqrtf(l);
  }
}

// ---------------------------------------------------------------------------
// Key coordinates y = P^T k.  grid = (ceil(N/64), BH), block = 256.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_key_coords(const __nv_bfloat16* __restrict__ K, int N, int R,
                                                   const float* __restrict__ proj, float* __restrict__ Y) {
  extern __shared__ __align__(16) unsigned char smem[];
  float* ps = reinterpret_cast<float*>(smem);  // [D][R]
  float* ks = ps + D * R;                      // [64][D+1]
  const int bh = blockIdx.y, n0 = blockIdx.x * 64, tid = threadIdx.x;
  for (int i = tid; i < D * R; i += blockDim.x) ps[i] = proj[(size_t)bh * D * R + i];
  const int nr = min(64, N - n0);
  const __nv_bfloat16* Kh = K + ((size_t)bh * N + n0) * D;
  for (int e = tid; e < nr * D; e += blockDim.x) {
    int r = e / D, c = e - r * D;
    ks[r * (D + 1) + c] = bf2f(Kh[e]);
  }
  __syncthreads();
  for (int e = tid; e < nr * R; e += blockDim.x) {
    int r = e / R, j = e - r * R;
    float acc = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) acc = fmaf(ks[r * (D + 1) + c], ps[c * R + j], acc);
    Y[((size_t)bh * N + n0 + r) * R + j] = acc;
  }
}

// ---------------------------------------------------------------------------
// Stable counting sort by label.  grid = BH, block = 1024, dynamic smem = (33 * G) ints.
// perm[pos] = original index; offsets[g] = first position.  Warp w owns the contiguous
// rows [w R, (w + 1) R) (R = ceil(N / 32)): it counts its labels, the counts are turned
// into each (warp, label)'s first position (label-major, then warp order, so equal labels
// keep their row order), and the warp places its rows walking them in order, 32 at a
// time (a label's rank among the 32 by __match_any_sync).  Three block barriers in all.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) k_group_sort(const int* __restrict__ labels, int N, int G,
                                                    int* __restrict__ perm, int* __restrict__ offsets,
                                                    int* err) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* total = reinterpret_cast<int*>(smem);  // [G]
  int* wcnt = total + G;                       // [32][G]: counts, then first positions
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int* lab = labels + (size_t)bh * N;
  const int R = (N + 31) / 32, r0 = warp * R, r1 = min(N, r0 + R);
  for (int e = tid; e < 33 * G; e += blockDim.x) total[e] = 0;
  __syncthreads();
  int* mine = wcnt + warp * G;
  for (int i0 = r0; i0 < r1; i0 += 32) {
    const int i = i0 + lane;
    int l = -1;
    if (i < r1) {
      l = lab[i];
      if (l < 0 || l >= G) { set_error(err, DERR_INDEX); l = -1; }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, l);
    if (l >= 0 && lane == __ffs(peers) - 1) mine[l] += __popc(peers);
  }
  __syncthreads();
  // first position of each (warp, label): offset of the label, then the earlier warps'
  if (tid < G) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcnt[w * G + tid];
      wcnt[w * G + tid] = run;
      run += c;
    }
    total[tid] = run;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int g = 0; g < G; ++g) {
      const int c = total[g];
      total[g] = run;
      offsets[(size_t)bh * (G + 1) + g] = run;
      run += c;
    }
    offsets[(size_t)bh * (G + 1) + G] = run;
  }
  __syncthreads();
  for (int i0 = r0; i0 < r1; i0 += 32) {
    const int i = i0 + lane;
    int l = i < r1 ? lab[i] : -1;
    if (l >= G || l < 0) l = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, l);
    if (l >= 0) {
      const int rank = __popc(peers & ((1u << lane) - 1));
      perm[(size_t)bh * N + total[l] + mine[l] + rank] = i;
    }
    __syncwarp();
    if (l >= 0 && lane == __ffs(peers) - 1) mine[l] += __popc(peers);
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// Query coordinates z = s Q C^T (fp32).  grid = (ceil(N/64), ceil(G/64), BH),
// block = 256, each thread a 4 x 4 output patch.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_query_coords(const __nv_bfloat16* __restrict__ Q, int N,
                                                     const float* __restrict__ C, int G, float scale,
                                                     float* __restrict__ Z) {
  __shared__ __align__(16) float qs[16][64 + 4];
  __shared__ __align__(16) float csm[16][64 + 4];
  const int bh = blockIdx.z, n0 = blockIdx.x * 64, g0 = blockIdx.y * 64, tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[4][4] = {};
  const __nv_bfloat16* Qh = Q + (size_t)bh * N * D;
  const float* Ch = C + (size_t)bh * G * D;
  for (int k0 = 0; k0 < D; k0 += 16) {
    for (int e = tid; e < 64 * 16; e += 256) {
      int r = e >> 4, k = e & 15;
      qs[k][r] = (n0 + r < N) ? bf2f(Qh[(size_t)(n0 + r) * D + k0 + k]) : 0.f;
      csm[k][r] = (g0 + r < G) ? Ch[(size_t)(g0 + r) * D + k0 + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float4 a = *reinterpret_cast<const float4*>(&qs[k][ty * 4]);
      float4 b = *reinterpret_cast<const float4*>(&csm[k][tx * 4]);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int n = n0 + ty * 4 + i;
    if (n >= N) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int g = g0 + tx * 4 + j;
      if (g < G) Z[((size_t)bh * N + n) * G + g] = scale * acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// Route selection (one CTA per head, block = 1024).
// Per query group a: non-empty K/V groups sorted by mass descending (ties -> lower
// g), sequential fp64 cumulative mass and int64 cumulative cost n_a * n_g.  The
// shared alpha is the largest value in [0, 1] whose total cost fits
// budget = density * N^2 - P * N (60 bisection steps in fp64); each group keeps
// the shortest prefix reaching alpha (at least one cell).  density >= 1 routes all
// non-empty cells.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int prefix_len(const double* cm, int L, double alpha) {
  int lo = 0, hi = L;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (cm[mid] >= alpha) hi = mid; else lo = mid + 1;
  }
  int n = lo < L ? lo + 1 : L;
  return n < 1 ? 1 : n;
}

__device__ long long block_sum_ll(long long v, long long* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  long long t = 0;
  for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) t += red[w];
  __syncthreads();
  return t;
}

// The 60 fp64 bisection steps on alpha are reproduced exactly: the first 50 run as 10
// rounds of 32-way multisection (the points lo + i (hi - lo) / 32 are dyadic with at most
// 50 bits, so exact, and the cost is monotone in alpha, so the round lands on the bracket
// five bisection steps would reach); the last 10 run as plain bisection, with the same
// rounding of mid = (lo + hi) / 2.  Per-row cumulative masses and K/V sizes live in shared
// memory (the cumulative mass is summed sequentially in rank order, as the definition
// reads); one warp evaluates one candidate alpha over all query groups.
// grid = BH, block = 1024, dynamic smem = route_select_smem(Gq, Gk).
//
// Frame-causal (qcum != NULL): the cost of cell (a, g) is its visible pairs,
// sum_f hist_q[a][f] * visk[g][f] with hist_q the per-frame query counts of group a, and the
// budget is density * V - P * V / N with V = sum_f (tokens of frame f) * (tokens of frames
// <= f).  Per-row cumulative costs are then at most n_a * N < 2^32 (N <= 65535).
__global__ void __launch_bounds__(1024) k_route_select(const float* __restrict__ mass, int N, int Gq, int Gk,
                                                      const int* __restrict__ qoff, const int* __restrict__ koff,
                                                      float density, int P, const int* __restrict__ qcum,
                                                      const int* __restrict__ visk, const int* __restrict__ fend,
                                                      int F, int* __restrict__ order,
                                                      unsigned char* __restrict__ route,
                                                      float* __restrict__ rho_exec, double* __restrict__ alpha_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const bool causal = qcum != nullptr;
  // rows padded to Gk + 1 entries: the lanes of a warp read different rows at once (the
  // per-lane prefix searches), and an unpadded 128-entry row stride puts them all in one bank
  const int GkP = Gk + 1;
  double* cmh = reinterpret_cast<double*>(smem);               // [Gq][GkP] cumulative mass in rank order
  // [Gq][GkP] cumulative K/V sizes (causal: cumulative cell costs)
  unsigned* pnk = reinterpret_cast<unsigned*>(cmh + (size_t)Gq * GkP);
  int* nk = reinterpret_cast<int*>(pnk + (size_t)Gq * GkP);     // [Gk]
  int* nq = nk + Gk;                                            // [Gq]
  int* misc = nq + Gq;                                          // [0] L, [1..32] round flags
  long long* red = reinterpret_cast<long long*>(                // [32], 8-byte aligned
      (reinterpret_cast<uintptr_t>(misc + 40) + 7) & ~(uintptr_t)7);
  const int bh = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* mh = mass + (size_t)bh * Gq * Gk;
  int* oh = order + (size_t)bh * Gq * Gk;
  unsigned char* rh = route + (size_t)bh * Gq * Gk;
  for (int g = tid; g < Gk; g += blockDim.x) nk[g] = koff[(size_t)bh * (Gk + 1) + g + 1] - koff[(size_t)bh * (Gk + 1) + g];
  for (int a = tid; a < Gq; a += blockDim.x) nq[a] = qoff[(size_t)bh * (Gq + 1) + a + 1] - qoff[(size_t)bh * (Gq + 1) + a];
  __syncthreads();
  if (warp == 0) {
    int c = 0;
    for (int g = lane; g < Gk; g += 32) c += nk[g] > 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) misc[0] = c;
  }
  // per row, one warp: bitonic sort of the row's groups (mass descending, ties to the lower
  // group; empty groups last) into the warp's scratch, then lane 0 takes the cumulative mass
  // (fp64, rank order, sequential) and cumulative K/V sizes
  float* wm = reinterpret_cast<float*>(red + 32) + warp * 2 * Gk;   // [Gk] masses in rank order
  unsigned* wn = reinterpret_cast<unsigned*>(wm + Gk);              // [Gk] their K/V sizes / cell costs
  const int* qc_h = causal ? qcum + (size_t)blockIdx.x * Gq * F : nullptr;
  const int* vk_h = causal ? visk + (size_t)blockIdx.x * Gk * F : nullptr;
  __syncthreads();
  const int L = misc[0];
  // The sort always spans 128 elements, four per lane (element e = 4 lane + q), so every
  // stage and exchange distance is a compile-time constant and the elements stay in
  // registers; positions g >= Gk carry (-inf, INT_MAX) and sort after every real group.
  for (int a = warp; a < Gq; a += blockDim.x / 32) {
    if (nq[a] == 0) continue;
    float km[4];
    int ki[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int g = lane * 4 + q;
      const bool on = g < Gk && nk[g] > 0;
      km[q] = on ? mh[a * Gk + g] : -INFINITY;
      ki[q] = g < Gk ? g : 0x7fffffff;
    }
    // "x before y" <=> x.m > y.m || (x.m == y.m && x.i < y.i)
#pragma unroll
    for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        if (j >= 4) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float om = __shfl_xor_sync(0xffffffffu, km[q], j >> 2);
            const int oi = __shfl_xor_sync(0xffffffffu, ki[q], j >> 2);
            const int e = lane * 4 + q;
            const bool first = ((e & k) == 0) == ((e & j) == 0);   // keep the earlier of the pair
            const bool mine_before = km[q] > om || (km[q] == om && ki[q] < oi);
            if (first != mine_before) { km[q] = om; ki[q] = oi; }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int q2 = q ^ j;
            if (q2 < q) continue;
            const int e = lane * 4 + q;
            const bool asc = (e & k) == 0;
            const bool q_before = km[q] > km[q2] || (km[q] == km[q2] && ki[q] < ki[q2]);
            if (asc != q_before) {
              const float tm = km[q]; km[q] = km[q2]; km[q2] = tm;
              const int ti = ki[q]; ki[q] = ki[q2]; ki[q2] = ti;
            }
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = lane * 4 + q;
      if (r < L) {
        oh[a * Gk + r] = ki[q];
        wm[r] = km[q];
        if (causal) {
          // visible pairs of cell (a, g): sum_f (queries of a in frame f) (keys of g in frames <= f)
          const int* qa = qc_h + (size_t)a * F;
          const int* vg = vk_h + (size_t)ki[q] * F;
          unsigned c = 0u;
          for (int f = 0; f < F; ++f) c += (unsigned)(qa[f] - (f > 0 ? qa[f - 1] : 0)) * (unsigned)vg[f];
          wn[r] = c;
        } else {
          wn[r] = (unsigned)nk[ki[q]];
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      // sequential in rank order; four ranks' inputs are fetched ahead of their sums
      double sm = 0.0;
      unsigned c = 0u;
      for (int r0 = 0; r0 < L; r0 += 4) {
        float m4[4];
        unsigned n4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          m4[u] = r0 + u < L ? wm[r0 + u] : 0.f;
          n4[u] = r0 + u < L ? wn[r0 + u] : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (r0 + u < L) {
            sm += (double)m4[u];
            c += n4[u];
            cmh[(size_t)a * GkP + r0 + u] = sm;
            pnk[(size_t)a * GkP + r0 + u] = c;
          }
        }
      }
    }
    __syncwarp();
  }
  __syncthreads();
  double visible = (double)N * (double)N;
  if (causal) {
    long long v = 0;
    for (int f = 0; f < F; ++f) v += (long long)(fend[f] - (f > 0 ? fend[f - 1] : 0)) * (long long)fend[f];
    visible = (double)v;
  }
  const double probe_pairs = causal ? (double)P * visible / (double)N : (double)P * (double)N;
  const double budget = (double)density * visible - probe_pairs;
  // routed pairs of row a when its prefix holds len cells
  auto row_cost = [&](int a, int len) -> long long {
    const long long c = (long long)pnk[(size_t)a * GkP + len - 1];
    return causal ? c : (long long)nq[a] * c;
  };
  // cost of alpha over the rows a = lane, lane + 32, ... (warp-wide sum)
  auto warp_cost = [&](double al) -> long long {
    long long t = 0;
    for (int a = lane; a < Gq; a += 32)
      if (nq[a] > 0) t += row_cost(a, prefix_len(cmh + (size_t)a * GkP, L, al));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return t;
  };
  double alpha;
  const bool all = density >= 1.0f;
  if (all) {
    alpha = 1.0;
  } else {
    double lo = 0.0, hi = 1.0;
    if (warp == 0) {
      const long long c0 = warp_cost(lo);
      if (lane == 0) misc[1] = (double)c0 <= budget ? 1 : 0;
    }
    __syncthreads();
    if (misc[1]) {
      for (int round = 0; round < 10; ++round) {
        const double w = (hi - lo) * (1.0 / 32.0);
        if (warp >= 1) {
          const long long c = warp_cost(lo + warp * w);
          if (lane == 0) misc[1 + warp] = (double)c <= budget ? 1 : 0;
        }
        __syncthreads();
        int k = 0;
        for (int i = 1; i < 32; ++i) k += misc[1 + i];
        __syncthreads();
        // monotone cost: the points that fit are exactly i = 1 .. k
        const double nlo = lo + k * w;
        hi = k < 31 ? lo + (k + 1) * w : hi;
        lo = nlo;
      }
      for (int it = 50; it < 60; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (warp == 0) {
          const long long c = warp_cost(mid);
          if (lane == 0) misc[1] = (double)c <= budget ? 1 : 0;
        }
        __syncthreads();
        if (misc[1]) lo = mid; else hi = mid;
        __syncthreads();
      }
    }
    alpha = lo;
  }
  for (int e = tid; e < Gq * Gk; e += blockDim.x) rh[e] = 0;
  __syncthreads();
  long long routed = 0;
  for (int a = tid; a < Gq; a += blockDim.x) {
    if (nq[a] == 0) continue;
    const int len = all ? L : prefix_len(cmh + (size_t)a * GkP, L, alpha);
    for (int r = 0; r < len; ++r) rh[a * Gk + oh[a * Gk + r]] = 1;
    routed += row_cost(a, len);
  }
  routed = block_sum_ll(routed, red);
  if (tid == 0) {
    rho_exec[bh] = (float)(((double)routed + probe_pairs) / visible);
    if (alpha_out) alpha_out[bh] = alpha;
  }
}

// ---------------------------------------------------------------------------
// Tile mask of the permuted layout.  grid = (T, BH), block = 256.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_block_mask(const unsigned char* __restrict__ route, int N, int Gq,
                                                   int Gk, int blk, const int* __restrict__ perm_q,
                                                   const int* __restrict__ label_q,
                                                   const int* __restrict__ perm_k,
                                                   const int* __restrict__ label_k,
                                                   unsigned char* __restrict__ bmask) {
  const int i = blockIdx.x, bh = blockIdx.y, T = (N + blk - 1) / blk;
  const int* pq = perm_q + (size_t)bh * N;
  const int* pk = perm_k + (size_t)bh * N;
  const int* lq = label_q + (size_t)bh * N;
  const int* lk = label_k + (size_t)bh * N;
  const int a0 = lq[pq[i * blk]], a1 = lq[pq[min(N, (i + 1) * blk) - 1]];
  const unsigned char* rh = route + (size_t)bh * Gq * Gk;
  for (int j = threadIdx.x; j < T; j += blockDim.x) {
    const int g0 = lk[pk[j * blk]], g1 = lk[pk[min(N, (j + 1) * blk) - 1]];
    unsigned char v = 0;
    for (int a = a0; a <= a1 && !v; ++a)
      for (int g = g0; g <= g1; ++g)
        if (rh[a * Gk + g]) { v = 1; break; }
    bmask[((size_t)bh * T + i) * T + j] = v;
  }
}

// ---------------------------------------------------------------------------
// Host-side launchers
// ---------------------------------------------------------------------------
static size_t sample_smem(int Ms, int D) {
  return (size_t)((Ms + 3) & ~3) * 4 + (size_t)64 * D * 4;
}

cudaError_t launch_sample_metric(const void* Q, int BH, int N, int D, int Ms, uint64_t seed, HeadMap hm,
                                 float* metric, int* sample_idx, int* err, cudaStream_t st) {
  size_t sm = sample_smem(Ms, D);
  if (D == 64) {
    cudaFuncSetAttribute(k_sample_metric<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_sample_metric<64><<<BH, 64 * 64 / 16, sm, st>>>((const __nv_bfloat16*)Q, N, Ms, seed, hm, metric, sample_idx,
                                                      err);
  } else {
    cudaFuncSetAttribute(k_sample_metric<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_sample_metric<128><<<BH, 128 * 128 / 16, sm, st>>>((const __nv_bfloat16*)Q, N, Ms, seed, hm, metric,
                                                         sample_idx, err);
  }
  return cudaGetLastError();
}

size_t metric_eigen_smem(int D, int R) {
  const size_t sc = D == 64 ? SymEigScratch<float, 64>::kCount : SymEigScratch<float, 128>::kCount;
  return ((size_t)D * (D + 1) + (size_t)D * (R + 1) + 64 + sc) * 4;
}

cudaError_t launch_metric_eigen(const float* metric, int BH, int D, int R, float* eigval, float* eigvec,
                                float* proj, float* lu, cudaStream_t st) {
  const size_t sm = metric_eigen_smem(D, R);
  if (D == 64) {
    cudaFuncSetAttribute(k_metric_eigen<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_metric_eigen<64><<<BH, 1024, sm, st>>>(metric, R, eigval, eigvec, proj, lu);
  } else {
    cudaFuncSetAttribute(k_metric_eigen<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_metric_eigen<128><<<BH, 1024, sm, st>>>(metric, R, eigval, eigvec, proj, lu);
  }
  return cudaGetLastError();
}

cudaError_t launch_key_coords(const void* K, int BH, int N, int D, int R, const float* proj, float* Y,
                              cudaStream_t st) {
  size_t sm = (size_t)(D * R + 64 * (D + 1)) * 4;
  dim3 grid(ceil_div(N, 64), BH);
  if (D == 64) {
    cudaFuncSetAttribute(k_key_coords<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_key_coords<64><<<grid, 256, sm, st>>>((const __nv_bfloat16*)K, N, R, proj, Y);
  } else {
    cudaFuncSetAttribute(k_key_coords<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_key_coords<128><<<grid, 256, sm, st>>>((const __nv_bfloat16*)K, N, R, proj, Y);
  }
  return cudaGetLastError();
}

int kmeans_dt(int Dc) {
  int dt = 8;
  while (dt < Dc) dt *= 2;
  return dt;
}

cudaError_t launch_group_sort(const int* labels, int BH, int N, int G, int* perm, int* offsets, int* err,
                              cudaStream_t st) {
  size_t sm = (size_t)33 * G * 4;
  cudaFuncSetAttribute(k_group_sort, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  k_group_sort<<<BH, 1024, sm, st>>>(labels, N, G, perm, offsets, err);
  return cudaGetLastError();
}

cudaError_t launch_query_coords(const void* Q, int BH, int N, int D, const float* C, int G, float scale,
                                float* Z, cudaStream_t st) {
  dim3 grid(ceil_div(N, 64), ceil_div(G, 64), BH);
  if (D == 64)
    k_query_coords<64><<<grid, 256, 0, st>>>((const __nv_bfloat16*)Q, N, C, G, scale, Z);
  else
    k_query_coords<128><<<grid, 256, 0, st>>>((const __nv_bfloat16*)Q, N, C, G, scale, Z);
  return cudaGetLastError();
}

size_t route_select_smem(int Gq, int Gk) {
  return (size_t)Gq * (Gk + 1) * 8 + (size_t)Gq * (Gk + 1) * 4 + (size_t)(Gk + Gq + 40) * 4 + 8 + 32 * 8 +
         (size_t)32 * 2 * Gk * 4;
}

cudaError_t launch_route_select(const float* mass, int BH, int N, int Gq, int Gk, const int* qoff,
                                const int* koff, float density, int P, const Causal& cz, int* order,
                                unsigned char* route, float* rho_exec, double* alpha, cudaStream_t st) {
  const size_t sm = route_select_smem(Gq, Gk);
  cudaFuncSetAttribute(k_route_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  k_route_select<<<BH, 1024, sm, st>>>(mass, N, Gq, Gk, qoff, koff, density, P, cz.on() ? cz.qcum : nullptr,
                                       cz.visk, cz.fend, cz.F, order, route, rho_exec, alpha);
  return cudaGetLastError();
}

// Identity matrix (d x d, fp32): the coordinate map of the semantic-grouping baseline.
__global__ void k_identity(float* __restrict__ A, int d) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < d * d; e += gridDim.x * blockDim.x)
    A[e] = (e / d == e % d) ? 1.f : 0.f;
}

cudaError_t launch_identity(float* A, int d, cudaStream_t st) {
  k_identity<<<ceil_div(d * d, 256), 256, 0, st>>>(A, d);
  return cudaGetLastError();
}

cudaError_t launch_block_mask(const unsigned char* route, int BH, int N, int Gq, int Gk, int blk,
                              const int* perm_q, const int* label_q, const int* perm_k, const int* label_k,
                              unsigned char* bmask, cudaStream_t st) {
  const int T = ceil_div(N, blk);
  k_block_mask<<<dim3(T, BH), 256, 0, st>>>(route, N, Gq, Gk, blk, perm_q, label_q, perm_k, label_k, bmask);
  return cudaGetLastError();
}

}  // namespace spr
