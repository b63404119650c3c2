// Leading eigenpairs of a small real symmetric matrix held in shared memory, computed by
// one CTA in fp64.
//
//   1. Householder reduction to tridiagonal form, A = Q T Q^T (Golub & Van Loan, "Matrix
//      Computations", Householder tridiagonalization): step k reflects column k below the
//      diagonal onto its first entry; the trailing block is updated as A -= v w^T + w v^T
//      with p = beta A v, w = p - (beta/2)(v^T p) v (a few threads per row for A v and the
//      update, v^T p reduced in the same pass).  The reflector v_k is kept in column k
//      below the diagonal.
//   2. Eigenvalues of T bracketed by multisection on the Sturm count (the number of negative
//      pivots of the LDL^T factorisation of T - x I), evaluated in fp32: each warp brackets one
//      eigenvalue and its 32 lanes test 32 interior points per step, so the bracket shrinks
//      33-fold a step, down to fp32 resolution (the shift of step 3).
//   3. Eigenvectors of T by inverse iteration: two solves with (T - mu I), tridiagonal LU with
//      partial pivoting, tiny pivots replaced by eps ||T||.  Eigenvalues closer than 1e-3 ||T||
//      form a cluster: their shifts are separated and their vectors re-orthogonalised by
//      modified Gram-Schmidt (the usual safeguard of inverse iteration).  The eigenvalue is
//      then the Rayleigh quotient of the unit vector.
//   4. Back-transformation z = Q y with the stored reflectors.
//
// Results: lam[j] = j-th largest eigenvalue, Z[:, j] (row stride ldz) its unit eigenvector.
#pragma once
#include <cfloat>

#include "common.cuh"

namespace spr {

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// number of eigenvalues of the tridiagonal (d, e2 = e^2, fp32 copies) not above x, in fp32:
// it only brackets the eigenvalue for the inverse iteration, whose Rayleigh quotient gives
// the fp64 value, so an fp32 bracket (and fast division) is enough
__device__ __forceinline__ int sturm_count_f32(const float* d, const float* e2, int n, float x, float pivmin) {
  float q = d[0] - x;
  if (fabsf(q) < pivmin) q = -pivmin;
  int c = q <= 0.f;
  for (int i = 1; i < n; ++i) {
    q = (d[i] - x) - __fdividef(e2[i - 1], q);
    if (fabsf(q) < pivmin) q = -pivmin;
    c += q <= 0.f;
  }
  return c;
}

// the same count in fp64 (for the last steps of the brackets)
__device__ __forceinline__ int sturm_count_f64(const double* d, const double* e2, int n, double x, double pivmin) {
  double q = d[0] - x;
  if (fabs(q) < pivmin) q = -pivmin;
  int c = q <= 0.0;
  for (int i = 1; i < n; ++i) {
    q = (d[i] - x) - e2[i - 1] / q;
    if (fabs(q) < pivmin) q = -pivmin;
    c += q <= 0.0;
  }
  return c;
}

// Solve (T - mu I) x = y in place (y[i * ys]), T = tridiag(e, d, e); u: 3n doubles of scratch.
// Single thread.  Pivots smaller than tol are replaced by +-tol.
__device__ inline void tri_shifted_solve(const double* d, const double* e, int n, double mu, double tol, double* y,
                                  int ys, double* u) {
  double r0 = d[0] - mu, r1 = n > 1 ? e[0] : 0.0, yi = y[0];
  for (int i = 0; i + 1 < n; ++i) {
    const double b = e[i], a1 = d[i + 1] - mu, c1 = (i + 2 < n) ? e[i + 1] : 0.0;
    const double yn = y[(i + 1) * ys];
    if (fabs(r0) >= fabs(b)) {
      const double l = r0 != 0.0 ? b / r0 : 0.0;
      u[3 * i] = r0; u[3 * i + 1] = r1; u[3 * i + 2] = 0.0;
      y[i * ys] = yi;
      r0 = a1 - l * r1; r1 = c1; yi = yn - l * yi;
    } else {  // row interchange
      const double l = r0 / b;
      u[3 * i] = b; u[3 * i + 1] = a1; u[3 * i + 2] = c1;
      y[i * ys] = yn;
      r0 = r1 - l * a1; r1 = -l * c1; yi = yi - l * yn;
    }
  }
  u[3 * (n - 1)] = r0; u[3 * (n - 1) + 1] = 0.0; u[3 * (n - 1) + 2] = 0.0;
  y[(n - 1) * ys] = yi;
  double x1 = 0.0, x2 = 0.0;
  for (int i = n - 1; i >= 0; --i) {
    double piv = u[3 * i];
    if (fabs(piv) < tol) piv = piv < 0.0 ? -tol : tol;
    const double x = (y[i * ys] - u[3 * i + 1] * x1 - u[3 * i + 2] * x2) / piv;
    y[i * ys] = x;
    x2 = x1; x1 = x;
  }
}

// deterministic start vector entry in [-1, 1)
__device__ __forceinline__ double start_entry(int i, int j) {
  uint64_t z = (uint64_t)(i + 1) * 0x9E3779B97F4A7C15ull + (uint64_t)(j + 1) * 0xD1B54A32D192ED03ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (double)(z >> 11) * (2.0 / 9007199254740992.0) - 1.0;
}

// Shared scratch (doubles) needed besides A and Z.
template <int N>
struct SymEigScratch {
  static constexpr int kDoubles = 7 * N + 3 * 64 + 8;
};

// A: N x N symmetric, row stride N + 1, overwritten (reflectors below the diagonal).
// Z: N x R output, row stride ldz (R <= 64).  lam: R outputs.  sc: SymEigScratch<N>::kDoubles
// doubles of shared memory.  lu: 3 N R doubles (shared or global) used by the solves.
// Called by every thread of the block; blockDim.x a multiple of 32, at most 1024.
template <int N>
__device__ inline void sym_top_eigen(double* A, int R, double* Z, int ldz, double* lam, double* sc, double* lu) {
  constexpr int LD = N + 1;
  constexpr int NC = (N + 31) / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  // threads per row of the trailing-block passes (a power of two <= 32) and rows per pass
  int TPR = 1;
  while (TPR < 32 && TPR * 2 * N <= (int)blockDim.x) TPR *= 2;
  const int RPP = blockDim.x / TPR;
  double* d = sc;            // [N]
  double* e = d + N;         // [N]  e[i] = T[i+1][i]
  double* e2 = e + N;        // [N]
  double* beta = e2 + N;     // [N]
  double* v = beta + N;      // [N]
  double* p = v + N;         // [N]
  float* d32 = reinterpret_cast<float*>(p + N);   // [N]
  float* e232 = d32 + N;                          // [N]
  double* shift = p + 2 * N; // [64]
  int* cstart = reinterpret_cast<int*>(shift + 64);  // [64]
  double* misc = shift + 64 + 64;                    // [64 + 8]: gl, gu, tnorm, pivmin
  double* red = misc + 8;                            // [32] per-warp partial sums (misc has 72)

  // ---- 1. tridiagonalisation
  for (int k = 0; k + 2 < N; ++k) {
    const int m = N - k - 1;  // trailing block: rows/cols k+1 .. N-1
    if (warp == 0) {
      double s = 0.0;
      for (int i = 1 + lane; i < m; i += 32) {
        const double x = A[(k + 1 + i) * LD + k];
        s += x * x;
      }
      s = warp_sum_f64(s);
      const double x0 = A[(k + 1) * LD + k];
      __syncwarp();  // every lane has read x0 before lane 0 overwrites it
      double b = 0.0, alpha = x0, v0 = 0.0;
      if (s > 0.0) {
        const double nrm = sqrt(x0 * x0 + s);
        alpha = x0 > 0.0 ? -nrm : nrm;
        v0 = x0 - alpha;
        b = 1.0 / (nrm * (nrm + fabs(x0)));  // 2 / (v^T v)
      }
      for (int i = lane; i < m; i += 32) {
        double vi = i == 0 ? v0 : A[(k + 1 + i) * LD + k];
        if (b == 0.0) vi = 0.0;
        v[i] = vi;
        A[(k + 1 + i) * LD + k] = vi;  // reflector kept for the back-transformation
      }
      if (lane == 0) { d[k] = A[k * LD + k]; e[k] = alpha; beta[k] = b; }
    }
    __syncthreads();
    const double b = beta[k];
    if (b != 0.0) {
      // p = b A v: TPR threads per row, each a strided part of the dot product, combined
      // with shuffles; the same pass sums v.p for kk (per warp, then over the warps)
      double vp = 0.0;
      for (int i0 = 0; i0 < m; i0 += RPP) {
        const int i = i0 + tid / TPR, sub = tid % TPR;
        double acc = 0.0;
        if (i < m) {
          const double* row = A + (k + 1 + i) * LD + (k + 1);
          for (int j = sub; j < m; j += TPR) acc += row[j] * v[j];
        }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (i < m && sub == 0) {
          const double pi = b * acc;
          p[i] = pi;
          vp += v[i] * pi;
        }
      }
      vp = warp_sum_f64(vp);
      if (lane == 0) red[warp] = vp;
      __syncthreads();
      double kk = lane < nw ? red[lane] : 0.0;
      kk = 0.5 * b * warp_sum_f64(kk);
      // A -= v w^T + w v^T on the trailing block, w = p - kk v
      for (int i0 = 0; i0 < m; i0 += RPP) {
        const int i = i0 + tid / TPR, sub = tid % TPR;
        if (i < m) {
          const double vi = v[i], wi = p[i] - kk * vi;
          double* row = A + (k + 1 + i) * LD + (k + 1);
          for (int j = sub; j < m; j += TPR) row[j] -= vi * (p[j] - kk * v[j]) + wi * v[j];
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (N >= 2) {
      d[N - 2] = A[(N - 2) * LD + N - 2];
      e[N - 2] = A[(N - 1) * LD + N - 2];
      beta[N - 2] = 0.0;
    }
    d[N - 1] = A[(N - 1) * LD + N - 1];
    e[N - 1] = 0.0;
    beta[N - 1] = 0.0;
  }
  __syncthreads();
  // ---- Gershgorin bounds, ||T||, pivmin
  if (warp == 0) {
    double lo = DBL_MAX, hi = -DBL_MAX, me2 = 0.0;
    for (int i = lane; i < N; i += 32) {
      const double r = (i > 0 ? fabs(e[i - 1]) : 0.0) + (i + 1 < N ? fabs(e[i]) : 0.0);
      lo = fmin(lo, d[i] - r);
      hi = fmax(hi, d[i] + r);
      if (i + 1 < N) {
        e2[i] = e[i] * e[i];
        me2 = fmax(me2, e2[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      me2 = fmax(me2, __shfl_xor_sync(0xffffffffu, me2, o));
    }
    for (int i = lane; i < N; i += 32) {
      d32[i] = (float)d[i];
      e232[i] = i + 1 < N ? (float)e2[i] : 0.f;
    }
    if (lane == 0) {
      const double tn = fmax(fabs(lo), fabs(hi));
      const double pad = 4e-6 * tn + 1e-30;   // covers the fp32 rounding of the counts
      misc[0] = lo - pad;
      misc[1] = hi + pad;
      misc[2] = tn;
      misc[3] = fmax((double)FLT_MIN * fmax(1.0, me2), 1e-30 * tn);
      misc[4] = me2;
    }
  }
  __syncthreads();
  const double tnorm = misc[2];
  const float pivmin32 = (float)misc[3];
  const double pivmin64 = fmax(DBL_MIN * fmax(1.0, misc[4]), 1e-300);
  // ---- 2. eigenvalues (j-th largest = ascending index N-1-j)
  for (int j = warp; j < R; j += nw) {
    const int t = N - 1 - j;
    double a = misc[0], b = misc[1];
    for (int it = 0; it < 8; ++it) {
      if (b - a <= 2e-7 * fmax(fabs(a), fabs(b)) + 1e-7 * tnorm + 1e-30) break;
      const double x = a + (b - a) * (double)(lane + 1) * (1.0 / 33.0);
      const unsigned below = __ballot_sync(0xffffffffu, sturm_count_f32(d32, e232, N, (float)x, pivmin32) <= t);
      const int lo = below ? 31 - __clz(below) : -1;
      const double xlo = __shfl_sync(0xffffffffu, x, lo < 0 ? 0 : lo);
      const double xhi = __shfl_sync(0xffffffffu, x, lo < 31 ? lo + 1 : 31);
      if (lo >= 0) a = xlo;
      if (lo < 31) b = xhi;
    }
    // fp64 steps: an eigenvalue far below ||T|| (a weak direction) needs a bracket well
    // inside its gaps to its neighbours, which the fp32 count cannot resolve; widen the fp32
    // bracket by its own rounding first
    {
      const double pad = 4e-6 * tnorm + 1e-30;
      a -= pad;
      b += pad;
      for (int it = 0; it < 4; ++it) {
        if (b - a <= 4.0 * DBL_EPSILON * fmax(fabs(a), fabs(b)) + pivmin64 + 1e-300) break;
        const double x = a + (b - a) * (double)(lane + 1) * (1.0 / 33.0);
        const unsigned below = __ballot_sync(0xffffffffu, sturm_count_f64(d, e2, N, x, pivmin64) <= t);
        const int lo = below ? 31 - __clz(below) : -1;
        const double xlo = __shfl_sync(0xffffffffu, x, lo < 0 ? 0 : lo);
        const double xhi = __shfl_sync(0xffffffffu, x, lo < 31 ? lo + 1 : 31);
        if (lo >= 0) a = xlo;
        if (lo < 31) b = xhi;
      }
    }
    if (lane == 0) lam[j] = 0.5 * (a + b);
  }
  __syncthreads();
  // cluster starts and separated shifts (serial, R <= 64)
  if (tid == 0) {
    const double ctol = 1e-3 * tnorm, pertol = 10.0 * DBL_EPSILON * tnorm;
    for (int j = 0; j < R; ++j) {
      cstart[j] = (j > 0 && lam[j - 1] - lam[j] <= ctol) ? cstart[j - 1] : j;
      double mu = lam[j];
      if (j > 0 && cstart[j] != j && shift[j - 1] - mu < pertol) mu = shift[j - 1] - pertol;
      shift[j] = mu;
    }
  }
  __syncthreads();
  // ---- 3. inverse iteration (lane 0 of the warp solves; the warp normalises)
  const double tol = fmax(DBL_EPSILON * tnorm, 1e-300);
  for (int j = warp; j < R; j += nw) {
    for (int i = lane; i < N; i += 32) Z[i * ldz + j] = start_entry(i, j);
    __syncwarp();
    for (int rep = 0; rep < 2; ++rep) {
      if (lane == 0) tri_shifted_solve(d, e, N, shift[j], tol, Z + j, ldz, lu + (size_t)j * 3 * N);
      __syncwarp();
      double mx = 0.0;
      for (int i = lane; i < N; i += 32) mx = fmax(mx, fabs(Z[i * ldz + j]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const double sm = mx > 0.0 ? 1.0 / mx : 1.0;
      double nn = 0.0;
      for (int i = lane; i < N; i += 32) {
        const double z = Z[i * ldz + j] * sm;
        nn += z * z;
      }
      nn = warp_sum_f64(nn);
      const double sc2 = nn > 0.0 ? sm / sqrt(nn) : 0.0;
      for (int i = lane; i < N; i += 32) Z[i * ldz + j] *= sc2;
      __syncwarp();
    }
  }
  __syncthreads();
  // modified Gram-Schmidt inside clusters, in eigenvalue order
  for (int j = 1; j < R; ++j) {
    if (cstart[j] < j && warp == j % nw) {
      for (int i = cstart[j]; i < j; ++i) {
        double dd = 0.0;
        for (int r = lane; r < N; r += 32) dd += Z[r * ldz + i] * Z[r * ldz + j];
        dd = warp_sum_f64(dd);
        for (int r = lane; r < N; r += 32) Z[r * ldz + j] -= dd * Z[r * ldz + i];
        __syncwarp();
      }
      double nn = 0.0;
      for (int r = lane; r < N; r += 32) nn += Z[r * ldz + j] * Z[r * ldz + j];
      nn = warp_sum_f64(nn);
      const double s = nn > 0.0 ? 1.0 / sqrt(nn) : 0.0;
      for (int r = lane; r < N; r += 32) Z[r * ldz + j] *= s;
    }
    if (cstart[j] < j) __syncthreads();
  }
  // Rayleigh quotient, then 4. back-transformation, one warp per column
  for (int j = warp; j < R; j += nw) {
    double rq = 0.0;
    for (int i = lane; i < N; i += 32) {
      const double zi = Z[i * ldz + j];
      double ty = d[i] * zi;
      if (i > 0) ty += e[i - 1] * Z[(i - 1) * ldz + j];
      if (i + 1 < N) ty += e[i] * Z[(i + 1) * ldz + j];
      rq += zi * ty;
    }
    rq = warp_sum_f64(rq);
    if (lane == 0) lam[j] = rq;
    __syncwarp();
    for (int k = N - 3; k >= 0; --k) {
      const double b = beta[k];
      if (b == 0.0) continue;
      const int m = N - k - 1;
      double dd = 0.0;
      for (int i = lane; i < m; i += 32) dd += A[(k + 1 + i) * LD + k] * Z[(k + 1 + i) * ldz + j];
      dd = b * warp_sum_f64(dd);
      for (int i = lane; i < m; i += 32) Z[(k + 1 + i) * ldz + j] -= dd * A[(k + 1 + i) * LD + k];
      __syncwarp();
    }
  }
  __syncthreads();
}

}  // namespace spr
