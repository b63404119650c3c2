// Leading eigenpairs of a small real symmetric matrix held in shared memory, computed by
// one CTA in the precision T (float or double).
//
//   1. Householder reduction to tridiagonal form, A = Q T Q^T (Golub & Van Loan, "Matrix
//      Computations", Householder tridiagonalization): step k reflects column k below the
//      diagonal onto its first entry; the trailing block is updated as A -= v w^T + w v^T
//      with p = beta A v, w = p - (beta/2)(v^T p) v.  4 N threads work on it, four per row,
//      over the trailing block only, synchronised by a barrier of their own; every warp
//      forms the reflector itself, so a step is two barriers and no serial section.  The
//      reflector v_k is kept in column k below the diagonal of A.
//   2. Eigenvalues of T bracketed by multisection on the Sturm count (the number of negative
//      pivots of the LDL^T factorisation of T - x I), evaluated in fp32: each warp brackets one
//      eigenvalue and its 32 lanes test 32 interior points per step, so the bracket shrinks
//      33-fold a step, down to fp32 resolution.  In double precision a few more steps with
//      an fp64 count follow, for eigenvalues far below ||T||.
//   3. Eigenvectors of T by inverse iteration: two solves with (T - mu I), tridiagonal LU with
//      partial pivoting, tiny pivots replaced by eps ||T||, one eigenvector per lane.  Eigenvalues closer than a
//      cluster tolerance (1e-3 ||T|| in double, 1e-2 ||T|| in float, where independent
//      inverse iteration leaves vectors orthogonal only to about eps ||T|| / gap) form a
//      cluster: their shifts are separated and their vectors re-orthogonalised by modified
//      Gram-Schmidt (the usual safeguard of inverse iteration).  The eigenvalue is then the
//      Rayleigh quotient of the unit vector.
//   4. Back-transformation z = Q y with the stored reflectors, the columns in the lanes and
//      the rows in bands of registers across warps.
//
// Results: lam[j] = j-th largest eigenvalue, Z[:, j] (row stride ldz) its unit eigenvector.
#pragma once
#include <cfloat>

#include "common.cuh"

namespace spr {

template <typename T>
__device__ __forceinline__ T warp_sum_t(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_f64(double v) { return warp_sum_t<double>(v); }

__device__ __forceinline__ float sq_root(float x) { return sqrtf(x); }
__device__ __forceinline__ double sq_root(double x) { return sqrt(x); }

// number of eigenvalues of the tridiagonal (d, e2 = e^2, fp32 copies) not above x, in fp32:
// it brackets the eigenvalue for the inverse iteration, whose Rayleigh quotient gives the
// final value, so an fp32 bracket (and fast division) is enough
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

// the same count in fp64 (for the last steps of the brackets in double precision)
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

__device__ __forceinline__ float quot(float a, float b) { return __fdividef(a, b); }
__device__ __forceinline__ double quot(double a, double b) { return a / b; }

// Solve (T - mu I) x = y in place (y[i * ys]), T = tridiag(e, d, e); u: 3n scalars of scratch
// at stride us (entry q of row i at u[(3 i + q) us]).  Single thread.  Pivots smaller than tol
// are replaced by +-tol.  In float the quotients use the fast approximate division (a few
// ulps: inverse iteration only needs the direction).
template <typename T>
__device__ inline void tri_shifted_solve(const T* d, const T* e, int n, T mu, T tol, T* y, int ys, T* u, int us) {
  T r0 = d[0] - mu, r1 = n > 1 ? e[0] : T(0), yi = y[0];
  for (int i = 0; i + 1 < n; ++i) {
    const T b = e[i], a1 = d[i + 1] - mu, c1 = (i + 2 < n) ? e[i + 1] : T(0);
    const T yn = y[(i + 1) * ys];
    T* ui = u + (size_t)3 * i * us;
    if (fabs(r0) >= fabs(b)) {
      const T l = r0 != T(0) ? quot(b, r0) : T(0);
      ui[0] = r0; ui[us] = r1; ui[2 * us] = T(0);
      y[i * ys] = yi;
      r0 = a1 - l * r1; r1 = c1; yi = yn - l * yi;
    } else {  // row interchange
      const T l = quot(r0, b);
      ui[0] = b; ui[us] = a1; ui[2 * us] = c1;
      y[i * ys] = yn;
      r0 = r1 - l * a1; r1 = -l * c1; yi = yi - l * yn;
    }
  }
  T* un = u + (size_t)3 * (n - 1) * us;
  un[0] = r0; un[us] = T(0); un[2 * us] = T(0);
  y[(n - 1) * ys] = yi;
  T x1 = T(0), x2 = T(0);
  for (int i = n - 1; i >= 0; --i) {
    const T* ui = u + (size_t)3 * i * us;
    T piv = ui[0];
    if (fabs(piv) < tol) piv = piv < T(0) ? -tol : tol;
    const T x = quot(y[i * ys] - ui[us] * x1 - ui[2 * us] * x2, piv);
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

// Shared scratch (scalars of type T) needed besides A and Z.
template <typename T, int N>
struct SymEigScratch {
  static constexpr int kCount = 6 * N + (int)(8 * N / sizeof(T)) + 3 * 64 + 8 + 2 * 2 * 8 * 32;
};

// A: N x N symmetric, row stride N + 1, overwritten (reflectors below the diagonal).
// Z: N x R output, row stride ldz (R <= 64).  lam: R outputs.  sc: SymEigScratch<T, N>::kCount
// scalars of shared memory.  lu: 3 N R scalars (shared or global) used by the solves.  R <= 64.
// Called by every thread of the block; blockDim.x == NT (at least 4 N, N a multiple of 32;
// the tridiagonalisation uses named barrier 1).
template <typename T, int N, int NT = 1024>
__device__ inline void sym_top_eigen(T* A, int R, T* Z, int ldz, T* lam, T* sc, T* lu) {
  constexpr bool kF64 = sizeof(T) == 8;
  constexpr int LD = N + 1;
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  T* d = sc;                // [N]
  T* e = d + N;             // [N]  e[i] = T[i+1][i]
  T* e2 = e + N;            // [N]
  T* beta = e2 + N;         // [N]
  T* v = beta + N;          // [N]
  T* p = v + N;             // [N]
  float* d32 = reinterpret_cast<float*>(p + N);    // [N]
  float* e232 = d32 + N;                           // [N]
  T* shift = p + N + 8 * N / sizeof(T);            // [64]
  int* cstart = reinterpret_cast<int*>(shift + 64);  // [64]
  T* misc = shift + 128;                             // [8]: gl, gu, tnorm, pivmin, max e^2
  T* red = misc + 8;                                 // [32] per-warp partial sums, then
                                                     // [2][2][8][32] back-transformation sums

  // ---- 1. tridiagonalisation: 4 N worker threads, four per row (columns interleaved by
  // 4); warp w holds rows 32 (w / 4) + w % 4 + 4 r, r = 0..7, so with row stride N + 1 the
  // warp's 32 accesses of a step hit distinct banks.  Every warp forms the reflector of
  // column k itself from the column in A (no serial section), and the reflector stays in
  // column k of A (only its first entry, v0, is written).  Two barriers per step.
  constexpr int TW = 4 * N;   // worker threads (named barrier 1)
  static_assert(TW <= NT && N % 32 == 0, "worker threads");
  if (tid < TW) {
    const int s = lane & 3, i = 32 * (warp >> 2) + (warp & 3) + 4 * (lane >> 2);
    auto bar = [] { asm volatile("bar.sync 1, %0;" ::"n"(TW) : "memory"); };
    T* Ai = A + i * LD;
    for (int k = 0; k + 2 < N; ++k) {
      const int m = N - k - 1;  // trailing block: rows/cols k+1 .. N-1
      // the reflector of column k (every warp; the column is final after step k - 1)
      T s2 = T(0);
      for (int r = 1 + lane; r < m; r += 32) {
        const T x = A[(k + 1 + r) * LD + k];
        s2 += x * x;
      }
      s2 = warp_sum_t<T>(s2);
      const T x0 = A[(k + 1) * LD + k];
      T b = T(0), alpha = x0, v0 = T(0);
      if (s2 > T(0)) {
        const T nrm = sq_root(x0 * x0 + s2);
        alpha = x0 > T(0) ? -nrm : nrm;
        v0 = x0 - alpha;
        b = T(1) / (nrm * (nrm + fabs(x0)));  // 2 / (v^T v)
      }
      if (tid == 0) { d[k] = A[k * LD + k]; e[k] = alpha; beta[k] = b; }
      if (b == T(0)) continue;   // uniform: the column is already reduced
      // v_j = A[j][k] for j > k + 1, v0 for j = k + 1, 0 above
      auto vj_of = [&](int j) -> T { return j == k + 1 ? v0 : A[j * LD + k]; };
      const T vi = i > k ? vj_of(i) : T(0);
      // p = b A v on the trailing block, v.p for kk
      T acc = T(0);
      if (i > k) {
        T a0 = T(0), a1 = T(0);
        int j = k + 1 + s;
        for (; j + 4 < N; j += 8) {
          a0 += Ai[j] * vj_of(j);
          a1 += Ai[j + 4] * vj_of(j + 4);
        }
        if (j < N) a0 += Ai[j] * vj_of(j);
        acc = a0 + a1;
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      const T pi = i > k ? b * acc : T(0);
      if (s == 0) p[i] = pi;
      T vp = warp_sum_t<T>(s == 0 ? vi * pi : T(0));
      if (lane == 0) red[warp] = vp;
      bar();
      T kk = lane < TW / 32 ? red[lane] : T(0);
      kk = T(0.5) * b * warp_sum_t<T>(kk);
      // A -= v w^T + w v^T on the trailing block, w = p - kk v
      if (i > k) {
        const T wi = pi - kk * vi;
        int j = k + 1 + s;
        for (; j + 4 < N; j += 8) {
          const T v0j = vj_of(j), v1j = vj_of(j + 4);
          const T p0 = p[j], p1 = p[j + 4];
          const T a0 = Ai[j], a1 = Ai[j + 4];
          Ai[j] = a0 - (vi * (p0 - kk * v0j) + wi * v0j);
          Ai[j + 4] = a1 - (vi * (p1 - kk * v1j) + wi * v1j);
        }
        if (j < N) {
          const T vj = vj_of(j);
          Ai[j] -= vi * (p[j] - kk * vj) + wi * vj;
        }
      }
      // every thread has read column k and x0: the reflector's first entry replaces x0
      bar();
      if (i == k + 1 && s == 0) Ai[k] = v0;
    }
    if (tid == 0) {
      if (N >= 2) {
        d[N - 2] = A[(N - 2) * LD + N - 2];
        e[N - 2] = A[(N - 1) * LD + N - 2];
        beta[N - 2] = T(0);
      }
      d[N - 1] = A[(N - 1) * LD + N - 1];
      e[N - 1] = T(0);
      beta[N - 1] = T(0);
    }
  }
  __syncthreads();
  // ---- Gershgorin bounds, ||T||, pivmin
  if (warp == 0) {
    T lo = kF64 ? (T)DBL_MAX : (T)FLT_MAX, hi = -lo, me2 = T(0);
    for (int i = lane; i < N; i += 32) {
      const T r = (i > 0 ? fabs(e[i - 1]) : T(0)) + (i + 1 < N ? fabs(e[i]) : T(0));
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
      const T tn = fmax(fabs(lo), fabs(hi));
      const T pad = T(4e-6) * tn + T(1e-30);   // covers the fp32 rounding of the counts
      misc[0] = lo - pad;
      misc[1] = hi + pad;
      misc[2] = tn;
      misc[3] = (T)fmax((double)FLT_MIN * fmax(1.0, (double)me2), 1e-30 * (double)tn);
      misc[4] = me2;
    }
  }
  __syncthreads();
  const T tnorm = misc[2];
  const float pivmin32 = (float)misc[3];
  // ---- 2. eigenvalues (j-th largest = ascending index N-1-j)
  for (int j = warp; j < R; j += NW) {
    const int t = N - 1 - j;
    T a = misc[0], b = misc[1];
    for (int it = 0; it < 8; ++it) {
      if (b - a <= T(2e-7) * fmax(fabs(a), fabs(b)) + T(1e-7) * tnorm + T(1e-30)) break;
      const T x = a + (b - a) * (T)(lane + 1) * (T(1) / T(33));
      const unsigned below = __ballot_sync(0xffffffffu, sturm_count_f32(d32, e232, N, (float)x, pivmin32) <= t);
      const int lo = below ? 31 - __clz(below) : -1;
      const T xlo = __shfl_sync(0xffffffffu, x, lo < 0 ? 0 : lo);
      const T xhi = __shfl_sync(0xffffffffu, x, lo < 31 ? lo + 1 : 31);
      if (lo >= 0) a = xlo;
      if (lo < 31) b = xhi;
    }
    if constexpr (kF64) {
      // fp64 steps: an eigenvalue far below ||T|| (a weak direction) needs a bracket well
      // inside its gaps to its neighbours, which the fp32 count cannot resolve; widen the
      // fp32 bracket by its own rounding first
      const double pivmin64 = fmax(DBL_MIN * fmax(1.0, (double)misc[4]), 1e-300);
      const double pad = 4e-6 * tnorm + 1e-30;
      a -= pad;
      b += pad;
      for (int it = 0; it < 4; ++it) {
        if (b - a <= 4.0 * DBL_EPSILON * fmax(fabs(a), fabs(b)) + pivmin64 + 1e-300) break;
        const double x = a + (b - a) * (double)(lane + 1) * (1.0 / 33.0);
        const unsigned below = __ballot_sync(0xffffffffu, sturm_count_f64((const double*)d, (const double*)e2, N, x,
                                                                          pivmin64) <= t);
        const int lo = below ? 31 - __clz(below) : -1;
        const double xlo = __shfl_sync(0xffffffffu, x, lo < 0 ? 0 : lo);
        const double xhi = __shfl_sync(0xffffffffu, x, lo < 31 ? lo + 1 : 31);
        if (lo >= 0) a = xlo;
        if (lo < 31) b = xhi;
      }
    }
    if (lane == 0) lam[j] = T(0.5) * (a + b);
  }
  __syncthreads();
  // cluster starts and separated shifts (serial, R <= 64)
  if (tid == 0) {
    const T eps = kF64 ? (T)DBL_EPSILON : (T)FLT_EPSILON;
    const T ctol = (kF64 ? T(1e-3) : T(1e-2)) * tnorm, pertol = T(10) * eps * tnorm;
    for (int j = 0; j < R; ++j) {
      cstart[j] = (j > 0 && lam[j - 1] - lam[j] <= ctol) ? cstart[j - 1] : j;
      T mu = lam[j];
      if (j > 0 && cstart[j] != j && shift[j - 1] - mu < pertol) mu = shift[j - 1] - pertol;
      shift[j] = mu;
    }
  }
  __syncthreads();
  // ---- 3. inverse iteration, one eigenvector per lane (lane j of warp j / 32 solves for
  // column j; the solves are sequential recurrences, so 32 of them share one instruction
  // stream); lu is interleaved, entry q of row i of column j at lu[(3 i + q) R + j]
  const T tol = fmax((kF64 ? (T)DBL_EPSILON : (T)FLT_EPSILON) * tnorm, kF64 ? (T)1e-300 : (T)1e-37);
  if (warp * 32 < R) {
    const int j = warp * 32 + lane;
    if (j < R) {
      T* zj = Z + j;
      for (int i = 0; i < N; ++i) zj[i * ldz] = (T)start_entry(i, j);
      for (int rep = 0; rep < 2; ++rep) {
        tri_shifted_solve<T>(d, e, N, shift[j], tol, zj, ldz, lu + j, R);
        T mx = T(0);
        for (int i = 0; i < N; ++i) mx = fmax(mx, fabs(zj[i * ldz]));
        const T sm = mx > T(0) ? T(1) / mx : T(1);
        T nn = T(0);
        for (int i = 0; i < N; ++i) {
          const T z = zj[i * ldz] * sm;
          nn += z * z;
        }
        const T sc2 = nn > T(0) ? sm / sq_root(nn) : T(0);
        for (int i = 0; i < N; ++i) zj[i * ldz] *= sc2;
      }
    }
  }
  __syncthreads();
  // modified Gram-Schmidt inside clusters, in eigenvalue order; one warp per cluster
  // (clusters are independent)
  {
    int ord = 0;
    for (int j0 = 0; j0 < R; ++j0) {
      if (cstart[j0] != j0) continue;
      if (ord++ % NW != warp) continue;
      for (int j = j0 + 1; j < R && cstart[j] == j0; ++j) {
        for (int i = j0; i < j; ++i) {
          T dd = T(0);
          for (int r = lane; r < N; r += 32) dd += Z[r * ldz + i] * Z[r * ldz + j];
          dd = warp_sum_t<T>(dd);
          for (int r = lane; r < N; r += 32) Z[r * ldz + j] -= dd * Z[r * ldz + i];
          __syncwarp();
        }
        T nn = T(0);
        for (int r = lane; r < N; r += 32) nn += Z[r * ldz + j] * Z[r * ldz + j];
        nn = warp_sum_t<T>(nn);
        const T s = nn > T(0) ? T(1) / sq_root(nn) : T(0);
        for (int r = lane; r < N; r += 32) Z[r * ldz + j] *= s;
        __syncwarp();
      }
    }
  }
  __syncthreads();
  // Rayleigh quotient of each column (one warp per column)
  for (int j = warp; j < R; j += NW) {
    T rq = T(0);
    for (int i = lane; i < N; i += 32) {
      const T zi = Z[i * ldz + j];
      T ty = d[i] * zi;
      if (i > 0) ty += e[i - 1] * Z[(i - 1) * ldz + j];
      if (i + 1 < N) ty += e[i] * Z[(i + 1) * ldz + j];
      rq += zi * ty;
    }
    rq = warp_sum_t<T>(rq);
    if (lane == 0) lam[j] = rq;
  }
  // ---- 4. back-transformation z = H_0 H_1 ... H_{N-3} y: the reflectors applied last to
  // first; column j in lane j % 32, the rows split into BW bands of BR rows (one warp per
  // band and column group); a reflector's dot products are summed over the bands through
  // shared memory (double-buffered: one barrier per reflector)
  {
    constexpr int BW = NT / 32 >= 16 ? 8 : NT / 64;   // row bands
    constexpr int BR = N / BW;
    static_assert(BR * BW == N, "row bands");
    T* part = red + 32;                               // [2][2][BW][32]
    const int band = warp % BW, cg = warp / BW, j = cg * 32 + lane;
    const bool active = cg < 2 && cg * 32 < R;
    const bool own = active && j < R;
    const int r0 = band * BR;
    T zr[BR];
    if (own) {
#pragma unroll
      for (int r = 0; r < BR; ++r) zr[r] = Z[(r0 + r) * ldz + j];
    }
    int par = 0;   // parity of the applied reflectors (skipped ones do not toggle it)
    for (int k = N - 3; k >= 0; --k) {
      const T b = beta[k];
      if (b == T(0)) continue;   // uniform
      T* pk = part + par * 2 * BW * 32;
      par ^= 1;
      if (active) {
        T dd = T(0);
#pragma unroll
        for (int r = 0; r < BR; ++r)
          if (r0 + r > k) dd += A[(r0 + r) * LD + k] * (own ? zr[r] : T(0));
        pk[(cg * BW + band) * 32 + lane] = dd;
      }
      __syncthreads();
      if (active) {
        T dd = T(0);
#pragma unroll
        for (int w = 0; w < BW; ++w) dd += pk[(cg * BW + w) * 32 + lane];
        dd *= b;
#pragma unroll
        for (int r = 0; r < BR; ++r)
          if (r0 + r > k) zr[r] -= dd * A[(r0 + r) * LD + k];
      }
    }
    if (own) {
#pragma unroll
      for (int r = 0; r < BR; ++r) Z[(r0 + r) * ldz + j] = zr[r];
    }
  }
  __syncthreads();
}

}  // namespace spr
