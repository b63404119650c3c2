// Exact probe rows, residual subspace, ridge fit and correction (gist.science
// technical summary, section 2.B; huashangw.com article, method walkthrough:
// 64 probe rows per head drawn evenly from every query group, ridge regression,
// correction inside the leading singular directions of the probe residuals).
#include <cuda.h>

#include "common.cuh"
#include "symeig.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace spr {

// ---------------------------------------------------------------------------
// Probe rows.  Allocation by water-filling over the query groups (every group with
// spare members gets floor(remaining / #open) per round; a share of 0 sends the
// leftovers one each to open groups by decreasing size, ties to the lower index);
// inside group a, alloc_a members drawn without replacement with the probe stream,
// groups in ascending order.  grid = BH, block = 256.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_probe_pick(const int* __restrict__ perm_q, const int* __restrict__ qoff,
                                                   int N, int Gq, int P, uint64_t seed, HeadMap hm,
                                                   int* __restrict__ probe_idx, int* __restrict__ probe_grp,
                                                   int* err) {
  extern __shared__ __align__(16) unsigned char smem[];
  int* size = reinterpret_cast<int*>(smem);  // [Gq]
  int* alloc = size + Gq;                     // [Gq]
  int* order = alloc + Gq;                    // [Gq] open groups by decreasing size
  int* draw = order + Gq;                     // [P]
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int* qo = qoff + (size_t)bh * (Gq + 1);
  for (int a = tid; a < Gq; a += blockDim.x) { size[a] = qo[a + 1] - qo[a]; alloc[a] = 0; }
  __syncthreads();
  for (int a = tid; a < Gq; a += blockDim.x) {
    int r = 0;
    for (int b = 0; b < Gq; ++b) r += (size[b] > size[a]) || (size[b] == size[a] && b < a);
    order[r] = a;
  }
  __syncthreads();
  if (tid == 0) {
    int remaining = P;
    while (remaining > 0) {
      int open = 0;
      for (int a = 0; a < Gq; ++a) open += alloc[a] < size[a];
      if (open == 0) break;
      int share = remaining / open;
      if (share == 0) {
        for (int r = 0; r < Gq && remaining > 0; ++r) {
          int a = order[r];
          if (alloc[a] < size[a]) { alloc[a] += 1; --remaining; }
        }
        break;
      }
      for (int a = 0; a < Gq; ++a) {
        if (alloc[a] >= size[a]) continue;
        int add = min(share, size[a] - alloc[a]);
        alloc[a] += add;
        remaining -= add;
      }
    }
    SplitMix64 g(stream_state(seed, hm.global(bh), PURPOSE_PROBES));
    int outp = 0;
    for (int a = 0; a < Gq; ++a) {
      const int m = alloc[a];
      if (m == 0) continue;
      // partial Fisher-Yates of m of the group's n members: offsets j_i = i + next() mod (n - i);
      // draw i takes what position j_i holds before it, replayed through the earlier swaps
      // (a position p >= t holds p before draw t unless an earlier draw t' swapped with it,
      // and then what position t' held before draw t'), so no swap map is kept
      const int n = size[a];
      for (int i = 0; i < m; ++i) draw[i] = i + (int)(g.next() % (uint64_t)(n - i));
      for (int i = 0; i < m; ++i) {
        int pos = draw[i], t = i;
        while (true) {
          int tp = -1;
          for (int k = t - 1; k >= 0; --k)
            if (draw[k] == pos) { tp = k; break; }
          if (tp < 0) break;
          pos = tp;
          t = tp;
        }
        probe_idx[(size_t)bh * P + outp] = perm_q[(size_t)bh * N + qo[a] + pos];
        probe_grp[(size_t)bh * P + outp] = a;
        ++outp;
      }
    }
    for (; outp < P; ++outp) { probe_idx[(size_t)bh * P + outp] = -1; probe_grp[(size_t)bh * P + outp] = -1; }
  }
}

constexpr int PR = 64;  // probe rows per split in the partial buffers

// ---------------------------------------------------------------------------
// Merge the key splits: for each probe row and accumulator (dense / routed), the split
// maxima M_s, sums L_s and unnormalised outputs O_s combine as
//   M = max_s M_s, L = sum_s L_s 2^(M_s - M), O = sum_s O_s 2^(M_s - M) / L   (s ascending).
// grid = (P, BH), block = D (one output column per thread).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_probe_combine(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml, int S, int P, int D,
                                                      float* __restrict__ o_dense, float* __restrict__ o_sparse,
                                                      float* __restrict__ lse_d, float* __restrict__ lse_s) {
  __shared__ float sml[64 * 4];   // [S][M_dense, L_dense, M_sparse, L_sparse]
  const int r = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  const float LN2 = 0.69314718055994531f;
  for (int e = threadIdx.x; e < S * 4; e += blockDim.x) {
    const int sidx = e >> 2, k = e & 3;
    sml[e] = part_ml[(((size_t)bh * S + sidx) * PR + r) * 4 + k];
  }
  __syncthreads();
  for (int acc = 0; acc < 2; ++acc) {
    float M = -INFINITY;
    for (int sidx = 0; sidx < S; ++sidx) M = fmaxf(M, sml[sidx * 4 + 2 * acc]);
    float L = 0.f, Ov = 0.f;
    if (M != -INFINITY) {
      for (int sidx = 0; sidx < S; ++sidx) {
        const float ms = sml[sidx * 4 + 2 * acc];
        if (ms == -INFINITY) continue;
        const float w = ex2f(ms - M);
        L += sml[sidx * 4 + 2 * acc + 1] * w;
        if (c < D) Ov += part_o[((((size_t)bh * S + sidx) * PR + r) * 2 + acc) * D + c] * w;
      }
    }
    if (c < D) (acc == 0 ? o_dense : o_sparse)[((size_t)bh * P + r) * D + c] = L > 0.f ? Ov / L : 0.f;
    if (c == 0) {
      float* dst = acc == 0 ? lse_d : lse_s;
      if (dst) dst[(size_t)bh * P + r] = L > 0.f ? (M + log2f(L)) * LN2 : -INFINITY;
    }
  }
}

// ---------------------------------------------------------------------------
// Residual subspace + ridge fit, one CTA per head (fp64 arithmetic).
//   R = O_dense - O_sparse (P x D); top eigenpairs u_i, sigma_i^2 of the Gram R R^T
//   (Householder + multisection + inverse iteration); v_i = R^T u_i normalised (zero when
//   sigma_i <= 1e-6 sigma_0); Y = R V_r (the probes' residual coordinates).  The map's
//   input X is either the probes' whole sparse output (full_input: the pages' R ~ b + xB
//   with only the correction restricted to the subspace) or that output projected on V_r.
//   Centred dual ridge W = Xc^T (Xc Xc^T + lam I)^-1 Yc, b = ybar - xbar W; in the
//   projected reading W_sub (r x r) is exported as W = V_r W_sub, so in both readings a
//   row's residual coordinates are x W (x the row's full sparse output).
// grid = BH, block = FIT_THREADS.
// ---------------------------------------------------------------------------
constexpr int FIT_THREADS = 1024;

template <int D>
struct FitLayout {
  // doubles: G [PR][PR+1] (Gram -> Cholesky -> W_sub), Z [PR][Rk+1], lam [64], eigen scratch,
  // X = max(3 PR Rk (solver scratch), (2 D + 2 PR) Rk (V_r, Y, X V_r, W)), xbar [D], ybar,
  // bsub, cs [64 each]; then floats Rm, Xm [PR][D]
  __host__ __device__ static size_t xsize(int Rk) {
    const size_t a = (size_t)3 * PR * Rk, b = (size_t)(2 * D + 2 * PR) * Rk;
    return a > b ? a : b;
  }
  static size_t doubles(int Rk) {
    return (size_t)PR * (PR + 1) + (size_t)PR * (Rk + 1) + 64 + SymEigScratch<double, PR>::kCount + xsize(Rk) + D + 3 * 64;
  }
  static size_t bytes(int Rk) { return doubles(Rk) * 8 + (size_t)2 * PR * D * 4; }
};

template <int D>
__global__ void __launch_bounds__(FIT_THREADS) k_probe_fit(const float* __restrict__ o_dense,
                                                  const float* __restrict__ o_sparse, int P, int Rk,
                                                  double lam, float* __restrict__ Vr_out,
                                                  float* __restrict__ W_out, float* __restrict__ bfull_out,
                                                  float* __restrict__ Bmat, float* __restrict__ sigma_out,
                                                  float* __restrict__ bsub_out, const int* __restrict__ probe_grp,
                                                  const int* __restrict__ qoff, int Gq, int full_input) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int LDP = PR + 1;
  const int ldz = Rk + 1;
  const size_t xsz = FitLayout<D>::xsize(Rk);
  double* G = reinterpret_cast<double*>(smem);    // [PR][LDP]  Gram, later Cholesky, later W
  double* Z = G + PR * LDP;                        // [PR][Rk+1] eigenvectors of R R^T
  double* ev = Z + PR * ldz;                       // [64] eigenvalues, descending
  double* esc = ev + 64;                           // eigen scratch
  double* X = esc + SymEigScratch<double, PR>::kCount;   // solver scratch, then V_r and Y
  double* Vr = X;                                  // [D][Rk]
  double* Y = Vr + D * Rk;                         // [PR][Rk] -> solution
  double* Xs = Y + PR * Rk;                        // [PR][Rk] probe sparse outputs in the subspace
  double* Wd = Xs + PR * Rk;                       // [D][Rk] W = V_r W_sub
  double* xbar = X + xsz;                          // [D] mean of X (projected reading: the first Rk)
  double* ybar = xbar + D;                         // [64]
  double* bsub = ybar + 64;                        // [64]
  double* cs = bsub + 64;                          // [64]
  float* Rm = reinterpret_cast<float*>(cs + 64);   // [PR][D]
  float* Xm = Rm + PR * D;                         // [PR][D]
  const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  // the Gram is padded to PR x PR with zero rows (P <= PR): padding adds zero eigenvalues only
#pragma unroll 4
  for (int e = tid; e < PR * D; e += nt) {
    const int r = e / D;
    float od = 0.f, os = 0.f;
    if (r < P) {
      od = o_dense[(size_t)bh * P * D + e];
      os = o_sparse[(size_t)bh * P * D + e];
    }
    Rm[e] = od - os;
    Xm[e] = os;
  }
  __syncthreads();
  for (int e = tid; e < PR * PR; e += nt) {
    const int i = e / PR, j = e - i * PR;
    if (j > i) continue;
    double s = 0.0;
    for (int c = 0; c < D; ++c) s += (double)Rm[i * D + c] * (double)Rm[j * D + c];
    G[i * LDP + j] = s;
    G[j * LDP + i] = s;
  }
  __syncthreads();
  sym_top_eigen<double, PR>(G, Rk, Z, ldz, ev, esc, X);
  // subspace basis: v_j = R^T u_j / ||R^T u_j|| for the j-th largest eigenvalue of R R^T
  // (in fp64 these are orthogonal to ~1e-10 whenever sigma_j > 1e-6 sigma_max; smaller
  // singular values give zero columns)
  const double smax = sqrt(fmax(ev[0], 0.0));
  for (int e = tid; e < D * Rk; e += nt) {
    const int c = e / Rk, j = e - c * Rk;
    const double sj = sqrt(fmax(ev[j], 0.0));
    double v = 0.0;
    if (smax > 0.0 && sj > 1e-6 * smax)
      for (int p = 0; p < PR; ++p) v += (double)Rm[p * D + c] * Z[p * ldz + j];
    Vr[c * Rk + j] = v;
  }
  __syncthreads();
  for (int j = tid; j < Rk; j += nt) {
    const double sj = sqrt(fmax(ev[j], 0.0));
    const bool keep = smax > 0.0 && sj > 1e-6 * smax;
    if (sigma_out) sigma_out[(size_t)bh * Rk + j] = keep ? (float)sj : 0.f;
    double nn = 0.0;
    for (int c = 0; c < D; ++c) nn += Vr[c * Rk + j] * Vr[c * Rk + j];
    cs[j] = nn > 0.0 ? 1.0 / sqrt(nn) : 0.0;
  }
  __syncthreads();
  for (int e = tid; e < D * Rk; e += nt) Vr[e] *= cs[e % Rk];
  __syncthreads();
  // probe weights (cs is free again): 1, or n_a / (probes of group a) normalised to mean 1
  double* wt = cs;
  for (int i = tid; i < P; i += nt) {
    double w = 1.0;
    if (probe_grp) {
      const int* pg = probe_grp + (size_t)bh * P;
      const int a = pg[i];
      int cnt = 0;
      for (int k = 0; k < P; ++k) cnt += pg[k] == a;
      const int* qo = qoff + (size_t)bh * (Gq + 1);
      w = (a >= 0 && a < Gq && cnt > 0) ? (double)(qo[a + 1] - qo[a]) / cnt : 1.0;
    }
    wt[i] = w;
  }
  __syncthreads();
  if (tid == 0) {
    double sw = 0.0;
    for (int i = 0; i < P; ++i) sw += wt[i];
    const double f = sw > 0.0 ? (double)P / sw : 1.0;
    for (int i = 0; i < P; ++i) wt[i] *= f;
  }
  __syncthreads();
  // Y = R Vr and Xs = X Vr (the probes' residuals and sparse outputs in the subspace), means
  for (int e = tid; e < P * Rk; e += nt) {
    const int p = e / Rk, j = e - p * Rk;
    double s = 0.0, t = 0.0;
    for (int c = 0; c < D; ++c) {
      s += (double)Rm[p * D + c] * Vr[c * Rk + j];
      if (!full_input) t += (double)Xm[p * D + c] * Vr[c * Rk + j];
    }
    Y[p * Rk + j] = s;
    Xs[p * Rk + j] = t;
  }
  __syncthreads();
  // weighted means (the weights average to 1), centred rows scaled by sqrt(weight)
  const int XD = full_input ? D : Rk;   // width of the map's input
  for (int j = tid; j < (XD > Rk ? XD : Rk); j += nt) {
    double s = 0.0, t = 0.0;
    for (int p = 0; p < P; ++p) {
      if (j < Rk) s += wt[p] * Y[p * Rk + j];
      if (j < XD) t += wt[p] * (full_input ? (double)Xm[p * D + j] : Xs[p * Rk + j]);
    }
    if (j < Rk) ybar[j] = s / P;
    if (j < XD) xbar[j] = t / P;
  }
  __syncthreads();
  for (int e = tid; e < P * Rk; e += nt) {
    const int p = e / Rk, j = e - p * Rk;
    const double sq = sqrt(wt[p]);
    Y[p * Rk + j] = (Y[p * Rk + j] - ybar[j]) * sq;
    if (!full_input) Xs[p * Rk + j] = (Xs[p * Rk + j] - xbar[j]) * sq;
  }
  __syncthreads();
  // A = Xc Xc^T + lam I  (into G), Xc = the centred input rows scaled by sqrt(weight)
  for (int e = tid; e < P * P; e += nt) {
    const int i = e / P, j = e - i * P;
    double s = 0.0;
    if (full_input) {
      for (int c = 0; c < D; ++c) s += ((double)Xm[i * D + c] - xbar[c]) * ((double)Xm[j * D + c] - xbar[c]);
      s *= sqrt(wt[i]) * sqrt(wt[j]);
    } else {
      for (int c = 0; c < Rk; ++c) s += Xs[i * Rk + c] * Xs[j * Rk + c];
    }
    G[i * LDP + j] = s + (i == j ? lam : 0.0);
  }
  __syncthreads();
  // Cholesky A = L L^T (lower triangle of G)
  for (int k = 0; k < P; ++k) {
    if (tid == 0) G[k * LDP + k] = sqrt(G[k * LDP + k]);
    __syncthreads();
    const double dkk = G[k * LDP + k];
    for (int i = k + 1 + tid; i < P; i += nt) G[i * LDP + k] /= dkk;
    __syncthreads();
    for (int e = tid; e < (P - k - 1) * (P - k - 1); e += nt) {
      const int i = k + 1 + e / (P - k - 1), j = k + 1 + e % (P - k - 1);
      if (j <= i) G[i * LDP + j] -= G[i * LDP + k] * G[j * LDP + k];
    }
    __syncthreads();
  }
  // solve L L^T Z = Yc, one right-hand side per thread
  for (int j = tid; j < Rk; j += nt) {
    for (int i = 0; i < P; ++i) {
      double s = Y[i * Rk + j];
      for (int k = 0; k < i; ++k) s -= G[i * LDP + k] * Y[k * Rk + j];
      Y[i * Rk + j] = s / G[i * LDP + i];
    }
    for (int i = P - 1; i >= 0; --i) {
      double s = Y[i * Rk + j];
      for (int k = i + 1; k < P; ++k) s -= G[k * LDP + i] * Y[k * Rk + j];
      Y[i * Rk + j] = s / G[i * LDP + i];
    }
  }
  __syncthreads();
  if (full_input) {
    // W = Xc^T Z (D x Rk), b = ybar - xbar W
    for (int e = tid; e < D * Rk; e += nt) {
      const int c = e / Rk, j = e - c * Rk;
      double s = 0.0;
      for (int p = 0; p < P; ++p) s += sqrt(wt[p]) * ((double)Xm[p * D + c] - xbar[c]) * Y[p * Rk + j];
      Wd[e] = s;
      W_out[(size_t)bh * D * Rk + e] = (float)s;
      Vr_out[(size_t)bh * D * Rk + e] = (float)Vr[c * Rk + j];
    }
    __syncthreads();
    for (int j = tid; j < Rk; j += nt) {
      double s = 0.0;
      for (int c = 0; c < D; ++c) s += xbar[c] * Wd[c * Rk + j];
      bsub[j] = ybar[j] - s;
      if (bsub_out) bsub_out[(size_t)bh * Rk + j] = (float)bsub[j];
    }
  } else {
    // W_sub = Xc^T Z (Rk x Rk, in the Cholesky region), b = ybar - xbar W_sub
    double* Ws = G;
    for (int e = tid; e < Rk * Rk; e += nt) {
      const int i = e / Rk, j = e - i * Rk;
      double s = 0.0;
      for (int p = 0; p < P; ++p) s += Xs[p * Rk + i] * Y[p * Rk + j];
      Ws[e] = s;
    }
    __syncthreads();
    for (int j = tid; j < Rk; j += nt) {
      double s = 0.0;
      for (int i = 0; i < Rk; ++i) s += xbar[i] * Ws[i * Rk + j];
      bsub[j] = ybar[j] - s;
      if (bsub_out) bsub_out[(size_t)bh * Rk + j] = (float)bsub[j];
    }
    // W = V_r W_sub (D x Rk): residual coordinates of a row are x W = (x V_r) W_sub
    for (int e = tid; e < D * Rk; e += nt) {
      const int c = e / Rk, j = e - c * Rk;
      double s = 0.0;
      for (int i = 0; i < Rk; ++i) s += Vr[c * Rk + i] * Ws[i * Rk + j];
      Wd[e] = s;
      W_out[(size_t)bh * D * Rk + e] = (float)s;
      Vr_out[(size_t)bh * D * Rk + e] = (float)Vr[c * Rk + j];
    }
  }
  __syncthreads();
  for (int c = tid; c < D; c += nt) {
    double s = 0.0;
    for (int j = 0; j < Rk; ++j) s += Vr[c * Rk + j] * bsub[j];
    bfull_out[(size_t)bh * D + c] = (float)s;
  }
  if (Bmat) {
    for (int e = tid; e < D * D; e += nt) {
      const int r = e / D, c = e - r * D;
      double s = 0.0;
      for (int j = 0; j < Rk; ++j) s += Wd[r * Rk + j] * Vr[c * Rk + j];
      Bmat[(size_t)bh * D * D + e] = (float)s;
    }
  }
}

// ---------------------------------------------------------------------------
// Correction on the tensor cores: O = x + b_full + x B with B = W V_r^T (d x d).
// Persistent: CTA c takes the global 128-row tiles [c per, (c+1) per) (tile i = row tile
// i mod T of head i / T).  When the CTA enters a head it forms B^T[n][k] = sum_j V_r[n][j]
// W[k][j] (fp32) and splits it into bf16 hi + lo (K-major tile).  Then a pipeline:
//   warp 17     (lane 0) loads the O_sparse tile (two TMA boxes of 128 rows x 64 columns)
//               into a three-deep ring
//   warp 16     (lane 0) issues x B_hi + x B_lo (exact bf16 products, fp32 accumulation)
//               into a double-buffered TMEM tile
//   warps 0-15  row r = TMEM lane r, column quarter q: x + b + xB -> bf16, written in place
//               over x in the tile's ring slot; then thread 0 stores the slot to O with
//               TMA (3D map [BH][N][d], so a head's ragged last tile is clipped at row N) and
//               frees the slot once the store has read it
// Every row of a tile is loaded before the tile's outputs are written, so O may alias
// O_sparse.
// ---------------------------------------------------------------------------
namespace rct {
constexpr int NT = 576;
constexpr int NEPI = 512;
constexpr int MMA_WARP = 16;
constexpr int LOAD_WARP = 17;
constexpr int XS = 3;
constexpr int kCtas = 148;
struct Bars {
  uint64_t xfull[XS], xempty[XS], tfull[2], tempty[2];
};
}  // namespace rct

template <int D>
__global__ void __launch_bounds__(rct::NT, 1)
    k_reconstruct_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmo, int N, int T,
                     int total, int per, int Rk,
                     const float* __restrict__ W, const float* __restrict__ Vr, const float* __restrict__ bfull,
                     __nv_bfloat16* __restrict__ O, int* err) {
  using namespace spr::tc;
  extern __shared__ __align__(1024) unsigned char smem_rc[];
  const uint32_t base = su32(smem_rc);
  if (base & 1023u) {
    if (threadIdx.x == 0) set_error(err, DERR_INDEX);
    return;
  }
  const int t0 = blockIdx.x * per, t1 = min(total, t0 + per);
  if (t0 >= t1) return;
  constexpr int XS = rct::XS;
  constexpr uint32_t kT = (uint32_t)128 * D * 2;   // X tile (128 rows)
  constexpr uint32_t kB = (uint32_t)D * D * 2;     // B^T tile (D rows)
  const uint32_t sX = base, sBh = base + XS * kT, sBl = sBh + kB;
  float* sb = reinterpret_cast<float*>(smem_rc + XS * kT + 2 * kB);   // [D]
  rct::Bars* bars = reinterpret_cast<rct::Bars*>(sb + D);
  int* sMisc = reinterpret_cast<int*>(bars + 1);   // [0] tmem, [1] abort
  volatile int* abort_flag = sMisc + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    sMisc[1] = 0;
    for (int b = 0; b < XS; ++b) {
      mbar_init(su32(&bars->xfull[b]), 1);
      mbar_init(su32(&bars->xempty[b]), 1);   // thread 0, once the tile's store has read the slot
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(su32(&bars->tfull[b]), 1);
      mbar_init(su32(&bars->tempty[b]), rct::NEPI);
    }
    fence_barrier_init();
  }
  if (warp == rct::MMA_WARP) {
    tc_alloc(su32(&sMisc[0]), 256);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(D >> 3) << 17) | (8u << 24);
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };
  int it = 0;
  bool ok = true;
  for (int s0 = t0; s0 < t1 && ok;) {
    const int bh = s0 / T;
    const int s1 = min(t1, (bh + 1) * T);
    const size_t head = (size_t)bh * N;
    // ---- B^T of this head (every role is idle here)
    __syncthreads();
    {
      // V_r [n][j] and W^T [j][k] staged in the (idle) X ring: D * Rk <= 64 * 65 floats each
      const float* Wh = W + (size_t)bh * D * Rk;
      const float* Vh = Vr + (size_t)bh * D * Rk;
      float* sV = reinterpret_cast<float*>(smem_rc);
      float* sWt = sV + D * Rk;
      for (int e = tid; e < D * Rk; e += rct::NT) {
        sV[e] = Vh[e];
        const int k = e / Rk, j = e - k * Rk;
        sWt[j * D + k] = Wh[e];
      }
      __syncthreads();
      for (int e = tid; e < D * D; e += rct::NT) {
        const int n = e / D, k = e - n * D;
        float acc = 0.f;
        for (int j = 0; j < Rk; ++j) acc = fmaf(sV[n * Rk + j], sWt[j * D + k], acc);
        const __nv_bfloat16 hi = __float2bfloat16(acc);
        const __nv_bfloat16 lo = __float2bfloat16(acc - __bfloat162float(hi));
        const uint32_t off = tile_off(n, k >> 3, D) + (k & 7) * 2;
        *reinterpret_cast<__nv_bfloat16*>(smem_rc + XS * kT + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(smem_rc + XS * kT + kB + off) = lo;
      }
      for (int c = tid; c < D; c += rct::NT) sb[c] = bfull[(size_t)bh * D + c];
    }
    fence_proxy_async();
    __syncthreads();
    if (warp == rct::LOAD_WARP) {
      if (lane == 0) {
        for (int i = s0; i < s1 && ok; ++i, ++it) {
          const int xb = it % XS, n0 = (i - bh * T) * 128;
          if (it >= XS) ok = wait(bars->xempty[xb], ((it / XS) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(su32(&bars->xfull[xb]), kT);
#pragma unroll
          for (int h = 0; h < D / 64; ++h)
            tma_load_2d(sX + xb * kT + h * 16384, &tmx, 64 * h, (int)(head + n0), su32(&bars->xfull[xb]));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      it = __shfl_sync(0xffffffffu, it, 0);
    } else if (warp == rct::MMA_WARP) {
      if (lane == 0) {
        for (int i = s0; i < s1 && ok; ++i, ++it) {
          const int b = it & 1, xb = it % XS;
          ok = wait(bars->xfull[xb], (it / XS) & 1) && (it < 2 || wait(bars->tempty[b], ((it >> 1) - 1) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
            const uint32_t ob = (k >> 2) * (D * 128) + (k & 3) * 32;
            tc_mma(tmem + 128 * b, sdesc(sX + xb * kT + ox, 16, 1024), sdesc(sBh + ob, 16, 1024), idesc,
                   k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t ox = (k >> 2) * (128 * 128) + (k & 3) * 32;
            const uint32_t ob = (k >> 2) * (D * 128) + (k & 3) * 32;
            tc_mma(tmem + 128 * b, sdesc(sX + xb * kT + ox, 16, 1024), sdesc(sBl + ob, 16, 1024), idesc, 1u);
          }
          tc_commit(su32(&bars->tfull[b]));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      it = __shfl_sync(0xffffffffu, it, 0);
    } else {
      const int qt = warp >> 2, r = (warp & 3) * 32 + lane;
      const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
      constexpr int CQ = D / 4;   // columns of this quarter
      for (int i = s0; i < s1 && ok; ++i, ++it) {
        const int b = it & 1, xb = it % XS, n0 = (i - bh * T) * 128;
        // xB ready; the X tile (read below) completed before it
        const bool good =
            __all_sync(0xffffffffu, wait(bars->tfull[b], (it >> 1) & 1) && wait(bars->xfull[xb], (it / XS) & 1));
        if (good) {
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < CQ; c0 += 16) {
            const int cb = qt * CQ + c0;
            uint32_t acc[16];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
                "tcgen05.wait::ld.sync.aligned;\n"
                : "=r"(acc[0]), "=r"(acc[1]), "=r"(acc[2]), "=r"(acc[3]), "=r"(acc[4]), "=r"(acc[5]), "=r"(acc[6]),
                  "=r"(acc[7]), "=r"(acc[8]), "=r"(acc[9]), "=r"(acc[10]), "=r"(acc[11]), "=r"(acc[12]),
                  "=r"(acc[13]), "=r"(acc[14]), "=r"(acc[15])
                : "r"(tmem + 128 * b + lane_off + cb)
                : "memory");
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint4 xv = *reinterpret_cast<const uint4*>(smem_rc + xb * kT + tile_off(r, (cb >> 3) + q, 128));
              const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 x = __bfloat1622float2(x2[e]);
                const int c = cb + q * 8 + 2 * e;
                w[q * 4 + e] = pack_bf16(x.x + sb[c] + __uint_as_float(acc[q * 8 + 2 * e]),
                                         x.y + sb[c + 1] + __uint_as_float(acc[q * 8 + 2 * e + 1]));
              }
            }
            // in place: this thread read exactly these 32 bytes of the slot above
            *reinterpret_cast<uint4*>(smem_rc + xb * kT + tile_off(r, cb >> 3, 128)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(smem_rc + xb * kT + tile_off(r, (cb >> 3) + 1, 128)) =
                make_uint4(w[4], w[5], w[6], w[7]);
          }
          tc_fence_before();
          mbar_arrive(su32(&bars->tempty[b]));
          fence_proxy_async();   // the slot's new contents, to the TMA store
        }
        // every epilogue thread passes this barrier once per tile, whatever its waits gave
        if (!bar_and(1, rct::NEPI, good)) { ok = false; break; }
        if (tid == 0) {
#pragma unroll
          for (int h = 0; h < D / 64; ++h) tma_store_3d(&tmo, sX + xb * kT + h * 16384, 64 * h, n0, bh);
          bulk_commit();
          bulk_wait_read_all();
          mbar_arrive(su32(&bars->xempty[xb]));
        }
      }
      if (tid == 0) bulk_wait_all();
    }
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    s0 = s1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == rct::MMA_WARP) tc_dealloc(tmem, 256);
}

__global__ void k_probe_scatter(const int* __restrict__ probe_idx, const float* __restrict__ o_dense, int N, int P,
                                int D, __nv_bfloat16* __restrict__ O) {
  const int bh = blockIdx.x;
  for (int e = threadIdx.x; e < P * D; e += blockDim.x) {
    const int p = e / D, c = e - p * D;
    const int row = probe_idx[(size_t)bh * P + p];
    if (row >= 0 && row < N) O[((size_t)bh * N + row) * D + c] = __float2bfloat16(o_dense[(size_t)bh * P * D + e]);
  }
}

// ---------------------------------------------------------------------------
// Route lists and q-tile work list.  grid = BH, block = 256 (one warp per group).
//   rlist[a][i] = i-th routed non-empty K/V group of query group a (ascending g)
//   rcum[a][i]  = key rows before it, rcum[a][cnt] = total routed rows
//   tiles       = (a, t) for every 128-row tile of every non-empty query group
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_worklist(const unsigned char* __restrict__ route,
                                                 const int* __restrict__ qoff, const int* __restrict__ koff,
                                                 int Gq, int Gk, int tile_rows, int max_tiles,
                                                 int* __restrict__ rlist, int* __restrict__ rcum,
                                                 int* __restrict__ rcnt, int2* __restrict__ tiles,
                                                 int* __restrict__ tile_count) {
  const int bh = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int* ko = koff + (size_t)bh * (Gk + 1);
  for (int a = warp; a < Gq; a += 8) {
    const unsigned char* rr = route + ((size_t)bh * Gq + a) * Gk;
    int* rl = rlist + ((size_t)bh * Gq + a) * Gk;
    int* rc = rcum + ((size_t)bh * Gq + a) * (Gk + 1);
    int cnt = 0, cum = 0;
    for (int g0 = 0; g0 < Gk; g0 += 32) {
      const int g = g0 + lane;
      const int sz = g < Gk ? ko[g + 1] - ko[g] : 0;
      const bool on = g < Gk && rr[g] && sz > 0;
      const unsigned m = __ballot_sync(0xffffffffu, on);
      // exclusive prefix of sizes over the lanes that are on
      int v = on ? sz : 0, incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (on) {
        const int pos = cnt + __popc(m & ((1u << lane) - 1));
        rl[pos] = g;
        rc[pos] = cum + incl - v;
      }
      cnt += __popc(m);
      cum += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      rc[cnt] = cum;
      rcnt[(size_t)bh * Gq + a] = cnt;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int* qo = qoff + (size_t)bh * (Gq + 1);
    int t = 0;
    for (int a = 0; a < Gq; ++a) {
      const int nt = (qo[a + 1] - qo[a] + tile_rows - 1) / tile_rows;
      for (int k = 0; k < nt && t < max_tiles; ++k) tiles[(size_t)bh * max_tiles + t++] = make_int2(a, k);
    }
    tile_count[bh] = t;
  }
}

// ---------------------------------------------------------------------------
cudaError_t launch_worklist(const unsigned char* route, const int* qoff, const int* koff, int BH, int Gq, int Gk,
                           int tile_rows, int max_tiles, int* rlist, int* rcum, int* rcnt, int2* tiles,
                           int* tile_count, cudaStream_t st) {
  k_worklist<<<BH, 256, 0, st>>>(route, qoff, koff, Gq, Gk, tile_rows, max_tiles, rlist, rcum, rcnt, tiles,
                                 tile_count);
  return cudaGetLastError();
}

cudaError_t launch_probe_pick(const int* perm_q, const int* qoff, int BH, int N, int Gq, int P, uint64_t seed,
                              HeadMap hm, int* probe_idx, int* probe_grp, int* err, cudaStream_t st) {
  size_t sm = (size_t)(3 * Gq + 64 + 8) * 4;
  cudaFuncSetAttribute(k_probe_pick, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  k_probe_pick<<<BH, 256, sm, st>>>(perm_q, qoff, N, Gq, P, seed, hm, probe_idx, probe_grp, err);
  return cudaGetLastError();
}

int probe_splits(int N) {
  int s = (N + 2047) / 2048;
  return s < 1 ? 1 : (s > 64 ? 64 : s);
}

cudaError_t launch_probe_attn(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk, int Gq,
                              int P, const int* probe_idx, const int* probe_grp, const int* label_k,
                              const unsigned char* route, float scale_log2, const Causal& cz, float* part_o,
                              float* part_ml, int* err, cudaStream_t st) {
  return launch_probe_tc(Q, K, V, BH, N, D, Gk, Gq, P, probe_idx, probe_grp, label_k, route, scale_log2,
                         probe_splits(N), cz, part_o, part_ml, err, st);
}

// Split-count-explicit variants (the key-split count S is chosen by the caller instead
// of probe_splits(N)); used by the entry point whose scratch has a fixed size.
cudaError_t launch_probe_attn_splits(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk,
                                     int Gq, int P, const int* probe_idx, const int* probe_grp, const int* label_k,
                                     const unsigned char* route, float scale_log2, int S, float* part_o,
                                     float* part_ml, int* err, cudaStream_t st) {
  return launch_probe_tc(Q, K, V, BH, N, D, Gk, Gq, P, probe_idx, probe_grp, label_k, route, scale_log2, S, Causal{},
                         part_o, part_ml, err, st);
}

cudaError_t launch_probe_combine_splits(const float* part_o, const float* part_ml, int BH, int S, int P, int D,
                                        float* o_dense, float* o_sparse, float* lse_d, float* lse_s,
                                        cudaStream_t st) {
  if (S > 64) return cudaErrorInvalidValue;
  k_probe_combine<<<dim3(P, BH), 128, 0, st>>>(part_o, part_ml, S, P, D, o_dense, o_sparse, lse_d, lse_s);
  return cudaGetLastError();
}

cudaError_t launch_probe_combine(const float* part_o, const float* part_ml, int BH, int N, int P, int D,
                                 float* o_dense, float* o_sparse, float* lse_d, float* lse_s, cudaStream_t st) {
  k_probe_combine<<<dim3(P, BH), 128, 0, st>>>(part_o, part_ml, probe_splits(N), P, D, o_dense, o_sparse, lse_d,
                                               lse_s);
  return cudaGetLastError();
}

size_t probe_fit_smem(int D, int Rk) { return D == 64 ? FitLayout<64>::bytes(Rk) : FitLayout<128>::bytes(Rk); }

cudaError_t launch_probe_fit(const float* o_dense, const float* o_sparse, int BH, int D, int P, int Rk,
                             double lam, float* Vr, float* W, float* bfull, float* Bmat, float* sigma,
                             float* bsub, const int* probe_grp, const int* qoff, int Gq, int full_input,
                             cudaStream_t st) {
  const size_t sm = probe_fit_smem(D, Rk);
  if (D == 64) {
    cudaFuncSetAttribute(k_probe_fit<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_probe_fit<64><<<BH, FIT_THREADS, sm, st>>>(o_dense, o_sparse, P, Rk, lam, Vr, W, bfull, Bmat, sigma, bsub,
                                                  probe_grp, qoff, Gq, full_input);
  } else {
    cudaFuncSetAttribute(k_probe_fit<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_probe_fit<128><<<BH, FIT_THREADS, sm, st>>>(o_dense, o_sparse, P, Rk, lam, Vr, W, bfull, Bmat, sigma, bsub,
                                                  probe_grp, qoff, Gq, full_input);
  }
  return cudaGetLastError();
}

cudaError_t launch_reconstruct(const void* Os, int BH, int N, int D, int Rk, const float* W, const float* Vr,
                               const float* bfull, void* O, cudaStream_t st) {
  const size_t sm = (size_t)rct::XS * 128 * D * 2 + 2 * (size_t)D * D * 2 + (size_t)D * 4 + sizeof(rct::Bars) + 16;
  const int T = ceil_div(N, 128), total = BH * T;
  const int grid = total < rct::kCtas ? total : rct::kCtas;
  const int per = ceil_div(total, grid);
  CUtensorMap tmx, tmo;
  cudaError_t e = make_tmap_bf16_rows(&tmx, Os, (unsigned long long)BH * N, D, 128);
  if (e == cudaSuccess) e = make_tmap_bf16_3d(&tmo, O, (unsigned long long)BH, (unsigned long long)N, D, 128);
  if (e != cudaSuccess) return e;
  if (D == 64) {
    cudaFuncSetAttribute(k_reconstruct_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_reconstruct_tc<64><<<grid, rct::NT, sm, st>>>(tmx, tmo, N, T, total, per, Rk, W, Vr, bfull, (__nv_bfloat16*)O,
                                                    nullptr);
  } else {
    cudaFuncSetAttribute(k_reconstruct_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    k_reconstruct_tc<128><<<grid, rct::NT, sm, st>>>(tmx, tmo, N, T, total, per, Rk, W, Vr, bfull, (__nv_bfloat16*)O,
                                                     nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_probe_scatter(const int* probe_idx, const float* o_dense, int BH, int N, int P, int D, void* O,
                                 cudaStream_t st) {
  k_probe_scatter<<<BH, 256, 0, st>>>(probe_idx, o_dense, N, P, D, (__nv_bfloat16*)O);
  return cudaGetLastError();
}

}  // namespace spr
