// Single-CTA cyclic Jacobi eigensolver for small symmetric matrices in shared memory.
//
// Parallel ordering: the n/2 disjoint rotations of one round of a round-robin
// tournament (player n-1 fixed, the others rotating) are applied together, rows
// first (A <- J^T A) then columns (A <- A J, V <- V J); each rotation zeroes its
// (p, q) entry (Golub & Van Loan, symmetric Schur decomposition).  A sweep is n-1
// rounds.  Sweeps stop when the off-diagonal Frobenius norm is at most tol times the
// diagonal one (for fp32 the rounding floor of that ratio is near sqrt(n) u ~ 1e-6 at
// n = 128, so fp32 callers use tol = 2e-5), or after max_sweeps.
#pragma once
#include "common.cuh"

namespace spr {

template <typename T>
__device__ __forceinline__ T sqrt_t(T x);
template <>
__device__ __forceinline__ float sqrt_t<float>(float x) { return sqrtf(x); }
template <>
__device__ __forceinline__ double sqrt_t<double>(double x) { return sqrt(x); }

// A, V: N x N with leading dimension N + 1; N even.  scratch: cs[N] (T), pr[N] (int),
// red[64] (T).  Called by every thread of the block (any block size <= 1024).
template <typename T, int N>
__device__ void jacobi_eigen(T* A, T* V, T* cs, int* pr, T* red, int max_sweeps, T tol) {
  constexpr int LD = N + 1;
  constexpr int M = N - 1;
  constexpr int WORK = (N / 2) * N;
  const int tid = threadIdx.x, nt = blockDim.x;
  for (int i = tid; i < N * N; i += nt) {
    const int r = i / N, c = i % N;
    V[r * LD + c] = (r == c) ? T(1) : T(0);
  }
  __syncthreads();
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    T off = 0, dia = 0;
    for (int i = tid; i < N * N; i += nt) {
      const int r = i / N, c = i % N;
      const T a = A[r * LD + c];
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
    for (int round = 0; round < M; ++round) {
      if (tid < N / 2) {
        int p, q;
        if (tid == 0) { p = round; q = N - 1; }
        else { p = (round + tid) % M; q = (round - tid + M) % M; }
        if (p > q) { const int t = p; p = q; q = t; }
        const T app = A[p * LD + p], aqq = A[q * LD + q], apq = A[p * LD + q];
        T c = 1, s = 0;
        if (apq != T(0)) {
          const T tau = (aqq - app) / (T(2) * apq);
          const T t = (tau >= T(0) ? T(1) : T(-1)) / (fabs(tau) + sqrt_t<T>(T(1) + tau * tau));
          c = T(1) / sqrt_t<T>(T(1) + t * t);
          s = t * c;
        }
        pr[2 * tid] = p; pr[2 * tid + 1] = q;
        cs[2 * tid] = c; cs[2 * tid + 1] = s;
      }
      __syncthreads();
      for (int w = tid; w < WORK; w += nt) {
        const int k = w / N, j = w % N;
        const int p = pr[2 * k], q = pr[2 * k + 1];
        const T c = cs[2 * k], s = cs[2 * k + 1];
        const T ap = A[p * LD + j], aq = A[q * LD + j];
        A[p * LD + j] = c * ap - s * aq;
        A[q * LD + j] = s * ap + c * aq;
      }
      __syncthreads();
      for (int w = tid; w < WORK; w += nt) {
        const int k = w / N, i = w % N;
        const int p = pr[2 * k], q = pr[2 * k + 1];
        const T c = cs[2 * k], s = cs[2 * k + 1];
        const T ap = A[i * LD + p], aq = A[i * LD + q];
        A[i * LD + p] = c * ap - s * aq;
        A[i * LD + q] = s * ap + c * aq;
        const T vp = V[i * LD + p], vq = V[i * LD + q];
        V[i * LD + p] = c * vp - s * vq;
        V[i * LD + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }
}

// rank[i] = position of eigenvalue i in descending order (ties -> lower index first).
template <typename T, int N>
__device__ void eigen_ranks(const T* A, int* rank) {
  constexpr int LD = N + 1;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const T li = A[i * LD + i];
    int r = 0;
    for (int j = 0; j < N; ++j) {
      const T lj = A[j * LD + j];
      r += (lj > li) || (lj == li && j < i);
    }
    rank[i] = r;
  }
  __syncthreads();
}

}  // namespace spr
