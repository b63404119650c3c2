// sparsepr_probe_fit_noalloc: the probe + fit call with its scratch memory in a fixed,
// library-owned device array instead of a caller-provided workspace.
//
// Who needs it: callers that cannot call cudaMalloc -- runtimes that plan their whole
// device memory at start-up and forbid allocation afterwards, and host code running
// where an allocation is not allowed (cudaMalloc can synchronize the device).  Such a
// caller still owns every input and output buffer; only the scratch moves.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes.  Every GPU that
// loads the library holds it until the process exits.  In host code the array's name is
// only a stand-in for the symbol, never a device address: the entry point looks up the
// real address with cudaGetSymbolAddress once per device (with that device current) and
// passes that pointer to the kernels.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)16 << 20;  // 16 MiB
__device__ __align__(256) unsigned char g_probe_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use and
// kept for the life of the process; a cudaDeviceReset of that device invalidates it).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_probe_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

struct ScratchPlan {
  size_t err, grp, o_sparse, lse_d, lse_s, part_o, part_ml, total;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Scratch regions for S key splits: the error word (cleared by every call), then buffers
// whose every byte is written before it is read.
ScratchPlan plan(const sparsepr_params& p, int S) {
  ScratchPlan L{};
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  const size_t BH = (size_t)p.B * p.H, P = p.n_probes, d = p.d;
  L.err = take(4);
  L.grp = take(BH * P * 4);
  L.o_sparse = take(BH * P * d * 4);
  L.lse_d = take(BH * P * 4);
  L.lse_s = take(BH * P * 4);
  L.part_o = take(BH * S * kProbeRowsPerCta * 2 * d * 4);
  L.part_ml = take(BH * S * kProbeRowsPerCta * 4 * 4);
  L.total = o;
  return L;
}

// After the fit: if any kernel of this call recorded a device error (a bounded wait that
// ran out, an index out of range, a failed draw), the fit may have read partial results
// the call did not write, so every head's b_full, Vr, W (and Bmat) become NaN.
__global__ void k_poison_on_error(const int* __restrict__ err, int D, int Rk, float* __restrict__ b_full,
                                  float* __restrict__ Vr, float* __restrict__ W, float* __restrict__ Bmat) {
  if (*(volatile const int*)err == 0) return;
  const float nan = __int_as_float(0x7fc00000);
  const int bh = blockIdx.x;
  for (int i = threadIdx.x; i < D; i += blockDim.x) b_full[(size_t)bh * D + i] = nan;
  for (int i = threadIdx.x; i < D * Rk; i += blockDim.x) {
    Vr[(size_t)bh * D * Rk + i] = nan;
    W[(size_t)bh * D * Rk + i] = nan;
  }
  if (Bmat)
    for (int i = threadIdx.x; i < D * D; i += blockDim.x) Bmat[(size_t)bh * D * D + i] = nan;
}

}  // namespace
}  // namespace spr

using namespace spr;

extern "C" sparsepr_status sparsepr_probe_fit_noalloc(const sparsepr_params* p, const void* Q, const void* K,
                                                      const void* V, const int* label_k, const int* perm_q,
                                                      const int* qoff, const unsigned char* route, int* probe_idx,
                                                      float* probe_o_dense, float* b_full, float* Vr, float* W,
                                                      float* Bmat, void* stream) {
  const sparsepr_status st0 = sparsepr_validate(p);
  if (st0 != SPARSEPR_OK) return st0;
  if (p->frame_id) {
    set_last_error("sparsepr_probe_fit_noalloc: frame-causal probes need the workspace entry point");
    return SPARSEPR_EUNSUPPORTED;
  }
  if (!Q || !K || !V || !label_k || !perm_q || !qoff || !route || !probe_idx || !probe_o_dense || !b_full ||
      !Vr || !W) {
    set_last_error("sparsepr_probe_fit_noalloc: a required pointer is NULL");
    return SPARSEPR_EINVAL;
  }
  // Q is read 16 bytes at a time and K, V through TMA: all three start on a 16-byte boundary
  if (((uintptr_t)Q | (uintptr_t)K | (uintptr_t)V) & 15u) {
    set_last_error("sparsepr_probe_fit_noalloc: Q, K and V must be 16-byte aligned");
    return SPARSEPR_EINVAL;
  }
  // Fewer key splits when the default count does not fit the fixed scratch.
  int S = probe_splits(p->N);
  while (S > 0 && plan(*p, S).total > kStaticScratchBytes) --S;
  if (S == 0) {
    set_last_error("sparsepr_probe_fit_noalloc: problem exceeds the 16 MiB static scratch");
    return SPARSEPR_EUNSUPPORTED;
  }
  const ScratchPlan L = plan(*p, S);
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) {
    set_last_error("sparsepr_probe_fit_noalloc: cudaGetSymbolAddress failed");
    return SPARSEPR_ECUDA;
  }
  char* sc = static_cast<char*>(base);
  int* err = reinterpret_cast<int*>(sc + L.err);
  int* grp = reinterpret_cast<int*>(sc + L.grp);
  float* osp = reinterpret_cast<float*>(sc + L.o_sparse);
  float* lsd = reinterpret_cast<float*>(sc + L.lse_d);
  float* lss = reinterpret_cast<float*>(sc + L.lse_s);
  float* part_o = reinterpret_cast<float*>(sc + L.part_o);
  float* part_ml = reinterpret_cast<float*>(sc + L.part_ml);
  cudaStream_t st = (cudaStream_t)stream;
  const int BH = p->B * p->H, N = p->N, d = p->d, P = p->n_probes;
  const float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)d);
  HeadMap hm;
  hm.H = p->H;
  hm.total = p->heads_total ? p->heads_total : p->H;
  hm.offset = p->head_offset;
  int launches = 0;
  auto step = [&](cudaError_t err_, const char* what) -> bool {
    ++launches;
    if (err_ != cudaSuccess) set_last_error(what);
    return err_ == cudaSuccess;
  };
  if (cudaMemsetAsync(err, 0, 4, st) != cudaSuccess) {
    set_last_error("sparsepr_probe_fit_noalloc: clearing the error word failed");
    return SPARSEPR_ECUDA;
  }
  if (!step(launch_probe_pick(perm_q, qoff, BH, N, p->n_qgroups, P, p->seed, hm, probe_idx, grp, err, st),
            "sparsepr_probe_fit_noalloc: probe pick launch failed") ||
      !step(launch_probe_attn_splits(Q, K, V, BH, N, d, p->n_kgroups, p->n_qgroups, P, probe_idx, grp, label_k,
                                     route, scale * 1.4426950408889634f, S, part_o, part_ml, err, st),
            "sparsepr_probe_fit_noalloc: probe attention launch failed") ||
      !step(launch_probe_combine_splits(part_o, part_ml, BH, S, P, d, probe_o_dense, osp, lsd, lss, st),
            "sparsepr_probe_fit_noalloc: probe combine launch failed") ||
      !step(launch_probe_fit(probe_o_dense, osp, BH, d, P, p->sub_rank, (double)p->ridge_lambda, Vr, W, b_full,
                             Bmat, nullptr, nullptr, p->fit_weighted ? grp : nullptr, qoff, p->n_qgroups,
                             p->fit_input == 0, st),
            "sparsepr_probe_fit_noalloc: fit launch failed")) {
    set_launch_count(launches);
    return SPARSEPR_ECUDA;
  }
  k_poison_on_error<<<BH, 256, 0, st>>>(err, d, p->sub_rank, b_full, Vr, W, Bmat);
  if (!step(cudaGetLastError(), "sparsepr_probe_fit_noalloc: error check launch failed")) {
    set_launch_count(launches);
    return SPARSEPR_ECUDA;
  }
  set_launch_count(launches);
  return SPARSEPR_OK;
}
