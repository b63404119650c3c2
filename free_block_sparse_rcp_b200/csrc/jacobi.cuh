// Single-CTA cyclic Jacobi eigensolver for small symmetric matrices in shared memory.
//
// Parallel ordering: the n/2 disjoint rotations of one round of a round-robin
// tournament (player n-1 fixed, the others rotating) are applied together, rows
// first (A <- J^T A) then columns (A <- A J, V <- V J); each rotation zeroes its
// (p, q) entry (Golub & Van Loan, symmetric Schur decomposition).  A sweep is n-1
// rounds; sweeps stop when the off-diagonal Frobenius norm is below tol times the
// diagonal norm, or after max_sweeps.
#pragma once
#include "common.cuh"

namespace spr {

template <typename T>
__device__ __forceinline__ T sqrt_t(T x);
template <>
__device__ __forceinline__ float sqrt_t<float>(float x) { return sqrtf(x); }
template <>
__device__ __forceinline__ double sqrt_t<double>(double x) { return sqrt(x); }

// A, V: n x n, leading dimension ld (>= n, odd preferred); n even, n <= 2*blockDim.x.
// scratch: cs[n] (T), pr[n] (int), red[2*32] (T).  Called by every thread of the block.
template <typename T>
__device__ void jacobi_eigen(T* A, T* V, int n, int ld, T* cs, int* pr, T* red, int max_sweeps,
                             T tol) {
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int i = tid; i < n * n; i += nt) {
    int r = i / n, c = i - r * n;
    V[r * ld + c] = (r == c) ? T(1) : T(0);
  }
  __syncthreads();
  const int m = n - 1;
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    T off = 0, dia = 0;
    for (int i = tid; i < n * n; i += nt) {
      int r = i / n, c = i - r * n;
      T a = A[r * ld + c];
      if (r == c) dia += a * a; else off += a * a;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      off += __shfl_xor_sync(0xffffffffu, off, o);
      dia += __shfl_xor_sync(0xffffffffu, dia, o);
    }
    if ((tid & 31) == 0) { red[tid >> 5] = off; red[32 + (tid >> 5)] = dia; }
    __syncthreads();
    off = 0; dia = 0;
    for (int w = 0; w < (nt + 31) / 32; ++w) { off += red[w]; dia += red[32 + w]; }
    __syncthreads();
    if (off <= tol * tol * dia) break;
    for (int round = 0; round < m; ++round) {
      if (tid < n / 2) {
        int p, q;
        if (tid == 0) { p = round; q = n - 1; }
        else { p = (round + tid) % m; q = (round - tid + m) % m; }
        if (p > q) { int t = p; p = q; q = t; }
        T app = A[p * ld + p], aqq = A[q * ld + q], apq = A[p * ld + q];
        T c = 1, s = 0;
        if (apq != T(0)) {
          T tau = (aqq - app) / (T(2) * apq);
          T t = (tau >= T(0) ? T(1) : T(-1)) / (fabs(tau) + sqrt_t<T>(T(1) + tau * tau));
          c = T(1) / sqrt_t<T>(T(1) + t * t);
          s = t * c;
        }
        pr[2 * tid] = p; pr[2 * tid + 1] = q;
        cs[2 * tid] = c; cs[2 * tid + 1] = s;
      }
      __syncthreads();
      const int work = (n / 2) * n;
      for (int w = tid; w < work; w += nt) {
        int k = w / n, j = w - k * n;
        int p = pr[2 * k], q = pr[2 * k + 1];
        T c = cs[2 * k], s = cs[2 * k + 1];
        T ap = A[p * ld + j], aq = A[q * ld + j];
        A[p * ld + j] = c * ap - s * aq;
        A[q * ld + j] = s * ap + c * aq;
      }
      __syncthreads();
      for (int w = tid; w < work; w += nt) {
        int k = w / n, i = w - k * n;
        int p = pr[2 * k], q = pr[2 * k + 1];
        T c = cs[2 * k], s = cs[2 * k + 1];
        T ap = A[i * ld + p], aq = A[i * ld + q];
        A[i * ld + p] = c * ap - s * aq;
        A[i * ld + q] = s * ap + c * aq;
        T vp = V[i * ld + p], vq = V[i * ld + q];
        V[i * ld + p] = c * vp - s * vq;
        V[i * ld + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
}

// rank[i] = position of eigenvalue i in descending order (ties -> lower index first).
template <typename T>
__device__ void eigen_ranks(const T* A, int n, int ld, int* rank) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    T li = A[i * ld + i];
    int r = 0;
    for (int j = 0; j < n; ++j) {
      T lj = A[j * ld + j];
      r += (lj > li) || (lj == li && j < i);
    }
    rank[i] = r;
  }
  __syncthreads();
}

}  // namespace spr
