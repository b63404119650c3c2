// Shared device helpers of the SparsePR CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sparsepr.h"

namespace spr {

// ---------------------------------------------------------------------------
// Device error codes written to the workspace error word (first writer wins).
// ---------------------------------------------------------------------------
enum DeviceError : int {
  DERR_NONE = 0,
  DERR_INDEX = 1,        // an index read from an input array was out of range
  DERR_WAIT_TIMEOUT = 2, // a bounded wait on an mbarrier ran out
  DERR_DRAW = 3,         // random draw map overflow
  DERR_NONFINITE = 4,    // non-finite value where the algorithm forbids one
  DERR_FRAMES = 5,       // frame ids out of [0, n_frames) or decreasing in token order
  DERR_CAPACITY = 6      // more k-means label corrections for 16 groups in one pass than the 2048 kept
};

__device__ __forceinline__ void set_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------------------
// SplitMix64 (Steele, Lea & Flood 2014): state += 0x9E3779B97F4A7C15, output =
// mix(state) with the two xor-shift-multiply rounds and a final xor-shift.
// Streams: state0 = mix(seed + 0xD1B54A32D192ED03 * (8*bh + purpose + 1)).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

struct SplitMix64 {
  uint64_t s;
  __device__ explicit SplitMix64(uint64_t state) : s(state) {}
  __device__ __forceinline__ uint64_t next() {
    s += 0x9E3779B97F4A7C15ull;
    return sm64_mix(s);
  }
};

enum Purpose : int { PURPOSE_QUERY_SAMPLE = 0, PURPOSE_KEY_KMEANS = 1, PURPOSE_QUERY_KMEANS = 2,
                     PURPOSE_PROBES = 3 };

__device__ __forceinline__ uint64_t stream_state(uint64_t seed, int bh, int purpose) {
  return sm64_mix(seed + 0xD1B54A32D192ED03ull * (uint64_t)(8ll * bh + purpose + 1));
}

// Head index of the random streams: a call over heads [offset, offset + H) of a layer with
// `total` heads per batch element numbers local head bh = b * H + h as b * total + offset + h,
// so a head-split call draws exactly the streams the unsplit call draws for those heads.
struct HeadMap {
  int H = 1, total = 1, offset = 0;
  __host__ __device__ int global(int bh) const { return (bh / H) * total + offset + bh % H; }
};

// Draw m distinct values of [0, n) by a partial Fisher-Yates shuffle (j_i = i + next() mod
// (n - i), swap positions i and j_i, out[i] = position i after the swap), block-cooperatively
// (every thread of the block calls it).  The k-th number of a SplitMix64 stream is
// mix(state + k * gamma), so the offsets j_i = i + (number i + 1) mod (n - i) of all m draws
// are computed in parallel into jbuf[m].  The swaps are then replayed per draw instead of in
// order: before draw t a position p >= t holds p unless an earlier draw t' < t swapped with
// it (j_t' = p), and then, for the last such t', the value position t' held before draw t'
// -- the same question one level down.  So out[i] (the value at position j_i before draw i)
// follows that chain backwards; draws rarely collide (m << n), so the chain is short.  The
// same out[] as the sequential swaps.  Returns false on every thread when 2 m exceeds cap
// (the callers' scratch bound).
__device__ inline bool draw_without_replacement_block(uint64_t state, int n, int m, int cap, int* out,
                                                      int* jbuf) {
  if (2 * m > cap) return false;
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    const uint64_t r = sm64_mix(state + 0x9E3779B97F4A7C15ull * (uint64_t)(i + 1));
    jbuf[i] = i + (int)(r % (uint64_t)(n - i));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < m; i += blockDim.x) {
    int p = jbuf[i], t = i;
    while (true) {
      int tp = -1;
      for (int k = t - 1; k >= 0; --k)
        if (jbuf[k] == p) { tp = k; break; }
      if (tp < 0) break;
      p = tp;
      t = tp;
    }
    out[i] = p;
  }
  __syncthreads();
  return true;
}

// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 2^x with the hardware approximation (ex2.approx, max error ~2 ulp).
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace spr
