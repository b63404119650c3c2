// Frame tables of the frame-causal mask (world-model rollout: a query of frame f sees the
// keys of frames <= f, intersected with the route).
//
// With frame ids nondecreasing in token order, and every group's members kept in ascending
// token order by the stable group sort, the members of a group that lie in frames <= f are
// a prefix of the group's permuted range.  Three small kernels turn that into tables:
//   fend[f]        tokens with frame <= f (the visible key prefix of a frame-f query in
//                  token order; also validates the ids),
//   cum[bh][g][f]  members of group g with frame <= f (K/V groups: the keys a frame-f
//                  query can see in g; query groups: the cumulative frame histogram),
//   the causal key stream of each query group: the keys of its routed K/V groups in
//                  frame-major order (frame 0 of every routed group, then frame 1, ...),
//                  with tlim[bh][a][f] = its length through frame f, so that the keys a
//                  frame-f query of group a may use are exactly the first tlim[a][f].
#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

__device__ __forceinline__ int clamp_frame(int f, int F) { return f < 0 ? 0 : (f >= F ? F - 1 : f); }

// One block: range and order check of frame_id, tokens per frame, prefix.
__global__ void __launch_bounds__(1024) k_frame_ends(const int* __restrict__ frame_id, int N, int F,
                                                     int* __restrict__ fend, int* err) {
  __shared__ int cnt[64];
  for (int f = threadIdx.x; f < F; f += blockDim.x) cnt[f] = 0;
  __syncthreads();
  bool bad = false;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int f = frame_id[i];
    if (f < 0 || f >= F || (i + 1 < N && frame_id[i + 1] < f)) bad = true;
    atomicAdd(&cnt[clamp_frame(f, F)], 1);
  }
  if (bad) set_error(err, DERR_FRAMES);
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int f = 0; f < F; ++f) {
      c += cnt[f];
      fend[f] = c;
    }
  }
}

// grid (G, BH), block 128: cum[bh][g][f] = members of group g (permuted range
// off[g] .. off[g+1]) whose frame is <= f.
__global__ void __launch_bounds__(128) k_group_frame_cum(const int* __restrict__ perm, const int* __restrict__ off,
                                                         const int* __restrict__ frame_id, int N, int G, int F,
                                                         int* __restrict__ cum, int* err) {
  __shared__ int cnt[64];
  const int g = blockIdx.x, bh = blockIdx.y;
  for (int f = threadIdx.x; f < F; f += blockDim.x) cnt[f] = 0;
  __syncthreads();
  const int* o = off + (size_t)bh * (G + 1);
  const int b0 = o[g], b1 = o[g + 1];
  for (int i = b0 + threadIdx.x; i < b1; i += blockDim.x) {
    const int t = perm[(size_t)bh * N + i];
    if (t < 0 || t >= N) {
      set_error(err, DERR_INDEX);
      continue;
    }
    atomicAdd(&cnt[clamp_frame(frame_id[t], F)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    int* dst = cum + ((size_t)bh * G + g) * F;
    for (int f = 0; f < F; ++f) {
      c += cnt[f];
      dst[f] = c;
    }
  }
}

// grid (Gq, BH), block 256.  Segment (f, i) of query group a = the keys of its i-th routed
// K/V group g that lie in frame f: permuted positions koff[g] + visk[g][f-1] .. koff[g] +
// visk[g][f].  Segments are laid out frame-major; klist[a][pos] = original key index.
constexpr int kStreamThreads = 256;
__global__ void __launch_bounds__(kStreamThreads) k_causal_stream(const int* __restrict__ rlist,
                                                                  const int* __restrict__ rcnt,
                                                                  const int* __restrict__ koff,
                                                                  const int* __restrict__ perm_k,
                                                                  const int* __restrict__ visk, int N, int Gq,
                                                                  int Gk, int F, int* __restrict__ klist,
                                                                  int* __restrict__ tlim, int* err) {
  extern __shared__ int sm_stream[];
  const int a = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int cnt = rcnt[(size_t)bh * Gq + a];
  const int* rl = rlist + ((size_t)bh * Gq + a) * Gk;
  const int* ko = koff + (size_t)bh * (Gk + 1);
  const int* vk = visk + (size_t)bh * Gk * F;
  int* pre = sm_stream;                       // [F * cnt + 1] exclusive prefix of segment lengths
  int* part = pre + (size_t)F * Gk + 1;       // [kStreamThreads]
  const int nseg = F * cnt;
  auto seg_len = [&](int s) -> int {
    const int f = s / cnt, g = rl[s - f * cnt];
    if (g < 0 || g >= Gk) return 0;
    const int* v = vk + (size_t)g * F;
    return v[f] - (f > 0 ? v[f - 1] : 0);
  };
  // block-wide exclusive scan: each thread owns a contiguous run of segments
  const int run = (nseg + kStreamThreads - 1) / kStreamThreads;
  const int s0 = min(nseg, tid * run), s1 = min(nseg, s0 + run);
  int local = 0;
  for (int s = s0; s < s1; ++s) local += seg_len(s);
  part[tid] = local;
  __syncthreads();
  if (tid == 0) {
    int c = 0;
    for (int t = 0; t < kStreamThreads; ++t) {
      const int v = part[t];
      part[t] = c;
      c += v;
    }
    pre[nseg] = c;
  }
  __syncthreads();
  {
    int c = part[tid];
    for (int s = s0; s < s1; ++s) {
      pre[s] = c;
      c += seg_len(s);
    }
  }
  __syncthreads();
  int* tl = tlim + ((size_t)bh * Gq + a) * F;
  for (int f = tid; f < F; f += kStreamThreads) tl[f] = cnt > 0 ? pre[(f + 1) * cnt] : 0;
  // copy: warp w takes segments w, w + 8, ...
  const int lane = tid & 31, warp = tid >> 5;
  int* dst = klist + ((size_t)bh * Gq + a) * N;
  const int* pk = perm_k + (size_t)bh * N;
  for (int s = warp; s < nseg; s += kStreamThreads / 32) {
    const int f = s / cnt, g = rl[s - f * cnt];
    if (g < 0 || g >= Gk) {
      if (lane == 0) set_error(err, DERR_INDEX);
      continue;
    }
    const int* v = vk + (size_t)g * F;
    const int src = ko[g] + (f > 0 ? v[f - 1] : 0);
    const int len = v[f] - (f > 0 ? v[f - 1] : 0);
    const int at = pre[s];
    if (src < 0 || len < 0 || src + len > N || at + len > N) {
      if (lane == 0) set_error(err, DERR_INDEX);
      continue;
    }
    for (int o = lane; o < len; o += 32) dst[at + o] = pk[src + o];
  }
}

}  // namespace

cudaError_t launch_frame_ends(const int* frame_id, int N, int F, int* fend, int* err, cudaStream_t st) {
  k_frame_ends<<<1, 1024, 0, st>>>(frame_id, N, F, fend, err);
  return cudaGetLastError();
}

cudaError_t launch_group_frame_cum(const int* perm, const int* off, const int* frame_id, int BH, int N, int G, int F,
                                   int* cum, int* err, cudaStream_t st) {
  k_group_frame_cum<<<dim3(G, BH), 128, 0, st>>>(perm, off, frame_id, N, G, F, cum, err);
  return cudaGetLastError();
}

size_t causal_stream_smem(int Gk, int F) { return ((size_t)F * Gk + 1 + kStreamThreads) * 4; }

cudaError_t launch_causal_stream(const int* rlist, const int* rcnt, const int* koff, const int* perm_k,
                                 const int* visk, int BH, int N, int Gq, int Gk, int F, int* klist, int* tlim,
                                 int* err, cudaStream_t st) {
  const size_t sm = causal_stream_smem(Gk, F);
  cudaError_t e = cudaFuncSetAttribute(k_causal_stream, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  k_causal_stream<<<dim3(Gq, BH), kStreamThreads, sm, st>>>(rlist, rcnt, koff, perm_k, visk, N, Gq, Gk, F, klist,
                                                           tlim, err);
  return cudaGetLastError();
}

}  // namespace spr
