// Internal launcher declarations of the SparsePR CUDA library.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace spr {

// Frame-causal inputs of the kernels below (all NULL / 0 without frame ids).
struct Causal {
  const int* frame_id = nullptr;   // [N]
  const int* fend = nullptr;       // [F] tokens with frame <= f
  const int* visk = nullptr;       // [BH][Gk][F] keys of group g with frame <= f
  const int* qcum = nullptr;       // [BH][Gq][F] queries of group a with frame <= f
  const int* klist = nullptr;      // [BH][Gq][N] causal key stream of each query group
  const int* tlim = nullptr;       // [BH][Gq][F] its length through frame f
  int F = 0;
  bool on() const { return frame_id != nullptr; }
};

// partition.cu
cudaError_t launch_sample_metric(const void* Q, int BH, int N, int D, int Ms, uint64_t seed, HeadMap hm,
                                 float* metric, int* sample_idx, int* err, cudaStream_t st);
size_t metric_eigen_smem(int D, int R);
cudaError_t launch_metric_eigen(const float* metric, int BH, int D, int R, float* eigval, float* eigvec,
                                float* proj, float* lu, cudaStream_t st);
cudaError_t launch_key_coords(const void* K, int BH, int N, int D, int R, const float* proj, float* Y,
                              cudaStream_t st);
int kmeans_dt(int Dc);
cudaError_t launch_group_sort(const int* labels, int BH, int N, int G, int* perm, int* offsets, int* err,
                              cudaStream_t st);
cudaError_t launch_query_coords(const void* Q, int BH, int N, int D, const float* C, int G, float scale,
                                float* Z, cudaStream_t st);
size_t route_select_smem(int Gq, int Gk);
cudaError_t launch_route_select(const float* mass, int BH, int N, int Gq, int Gk, const int* qoff,
                                const int* koff, float density, int P, const Causal& cz, int* order,
                                unsigned char* route, float* rho_exec, double* alpha, cudaStream_t st);
cudaError_t launch_identity(float* A, int d, cudaStream_t st);
cudaError_t launch_block_mask(const unsigned char* route, int BH, int N, int Gq, int Gk, int blk,
                              const int* perm_q, const int* label_q, const int* perm_k, const int* label_k,
                              unsigned char* bmask, cudaStream_t st);

// frames.cu: tables of the frame-causal mask (frame ids nondecreasing in token order)
constexpr int kMaxFrames = 64;
cudaError_t launch_frame_ends(const int* frame_id, int N, int F, int* fend, int* err, cudaStream_t st);
cudaError_t launch_group_frame_cum(const int* perm, const int* off, const int* frame_id, int BH, int N, int G, int F,
                                   int* cum, int* err, cudaStream_t st);
size_t causal_stream_smem(int Gk, int F);
cudaError_t launch_causal_stream(const int* rlist, const int* rcnt, const int* koff, const int* perm_k,
                                 const int* visk, int BH, int N, int Gq, int Gk, int F, int* klist, int* tlim,
                                 int* err, cudaStream_t st);
// tma_host.cu: 128-byte tensor map (CUtensorMap) of a row-major bf16 matrix for boxes of
// box_rows x 64 columns with 128B swizzle; rows past the end read as zeros.
cudaError_t make_tmap_bf16_rows(void* tmap, const void* base, unsigned long long rows, int cols, int box_rows);
cudaError_t make_tmap_bf16_3d(void* tmap, const void* base, unsigned long long outer, unsigned long long rows,
                              int cols, int box_rows);
struct alignas(64) TmapBlob {
  unsigned long long w[16];
};

// kmeans_tc.cu
int kmeans_gp(int G);
size_t centroid_weights_smem(int d, int D, int N);
size_t recheck_smem(int d, int D, int DT, int G, int N);
cudaError_t launch_seed_rows(const void* X, int BH, int N, int d, int G, uint64_t seed, HeadMap hm, int purpose,
                             float* m, int* init_out, int* err, cudaStream_t st);
// Persistent k-means assignment over segments of kKmeansSeg 128-row tiles of one head (head-
// major); CTA c takes a contiguous, balanced run of segments and leaves one partial-sum slot
// per segment, so the sums do not depend on the grid or on the number of heads.
constexpr int kKmeansCtas = 148;
constexpr int kKmeansSeg = 8;
struct KmPlan {
  int grid, T, SPH, nseg;
};
KmPlan kmeans_plan(int BH, int N);
// bytes of the segment slots of one k-means pass with GP (padded) groups and row width d
size_t kmeans_slots_bytes(int BH, int N, int GP, int d);
size_t assign_acc_smem(int D, int GP);
cudaError_t launch_centroid_weights(float* m, int BH, int G, int d, const float* A, size_t a_head, int sj, int sc,
                                    float a_scale, int D, int DT, int mode, const void* slots,
                                    const int* corr_count, const void* corr, const void* X, int N, float* nu,
                                    float* bias, float* wnorm, void* w_hi, void* w_lo, int* err, cudaStream_t st);
cudaError_t launch_assign_acc(const void* X, int BH, int N, int d, int G, const void* w_hi, const void* w_lo,
                              const float* bias, const float* wnorm, int* labels, int* trace, int* flag_seg,
                              int* flag_rows, void* slots, float* xnorm, int xnorm_store, int* err,
                              cudaStream_t st);
cudaError_t launch_assign_recheck(const void* X, int BH, int N, int d, const float* A, size_t a_head, int sj, int sc,
                                  float a_scale, int D, const float* nu, int G, const int* flag_seg,
                                  const int* flag_rows, int* labels, int* trace, int* corr_count, void* corr,
                                  cudaStream_t st);
size_t cell_mass_tc_smem(int D, int GP, int F);
cudaError_t launch_cell_mass_tc(const void* Q, int BH, int N, int d, int Gq, int Gk, const int* perm_q, const int* qoff,
                                const int* koff, const float* C, float scale, void* c1, void* c2, void* c3,
                                const Causal& cz, float* mass, int* err, cudaStream_t st);

// probe.cu
cudaError_t launch_worklist(const unsigned char* route, const int* qoff, const int* koff, int BH, int Gq, int Gk,
                           int tile_rows, int max_tiles, int* rlist, int* rcum, int* rcnt, int2* tiles,
                           int* tile_count, cudaStream_t st);
cudaError_t launch_probe_pick(const int* perm_q, const int* qoff, int BH, int N, int Gq, int P, uint64_t seed,
                              HeadMap hm, int* probe_idx, int* probe_grp, int* err, cudaStream_t st);
int probe_splits(int N);
size_t probe_tc_smem_bytes(int D, int Gk);
cudaError_t launch_probe_tc(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk, int Gq, int P,
                            const int* probe_idx, const int* probe_grp, const int* label_k, const unsigned char* route,
                            float scale_log2, int S, const Causal& cz, float* part_o, float* part_ml, int* err,
                            cudaStream_t st);
size_t probe_fit_smem(int D, int Rk);
cudaError_t launch_probe_attn(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk, int Gq,
                              int P, const int* probe_idx, const int* probe_grp, const int* label_k,
                              const unsigned char* route, float scale_log2, const Causal& cz, float* part_o,
                              float* part_ml, int* err, cudaStream_t st);
cudaError_t launch_probe_attn_splits(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk,
                                     int Gq, int P, const int* probe_idx, const int* probe_grp, const int* label_k,
                                     const unsigned char* route, float scale_log2, int S, float* part_o,
                                     float* part_ml, int* err, cudaStream_t st);
cudaError_t launch_probe_combine_splits(const float* part_o, const float* part_ml, int BH, int S, int P, int D,
                                        float* o_dense, float* o_sparse, float* lse_d, float* lse_s,
                                        cudaStream_t st);
cudaError_t launch_probe_combine(const float* part_o, const float* part_ml, int BH, int N, int P, int D,
                                 float* o_dense, float* o_sparse, float* lse_d, float* lse_s, cudaStream_t st);
// probe_grp / qoff: the weighted fit's probe groups and query group offsets (NULL: uniform);
// full_input: 1 = the map takes the whole sparse output row, 0 = its projection on V_r
cudaError_t launch_probe_fit(const float* o_dense, const float* o_sparse, int BH, int D, int P, int Rk,
                             double lam, float* Vr, float* W, float* bfull, float* Bmat, float* sigma,
                             float* bsub, const int* probe_grp, const int* qoff, int Gq, int full_input,
                             cudaStream_t st);
cudaError_t launch_reconstruct(const void* Os, int BH, int N, int D, int Rk, const float* W, const float* Vr,
                               const float* bfull, void* O, cudaStream_t st);
cudaError_t launch_probe_scatter(const int* probe_idx, const float* o_dense, int BH, int N, int P, int D, void* O,
                                 cudaStream_t st);

// attention
struct AttnArgs {
  const void* Q;
  const void* K;
  const void* V;
  int BH, N, D, Gq, Gk;
  const int* perm_q;
  const int* perm_k;
  const int* qoff;
  const int* koff;
  const int* rlist;
  const int* rcum;
  const int* rcnt;
  const int2* tiles;
  const int* tile_count;
  int max_tiles;
  float scale_log2;
  Causal cz;
  void* O;
  float* lse;
  int* err;
};
size_t attn_tc_smem_bytes(int D, int Gk);
cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, cudaStream_t st);
constexpr int kAttnTileRows = 256;   // query rows per attention work unit (two 128-row tiles)
constexpr int kProbeRowsPerCta = 64;  // probe rows per CTA of k_probe_attn (its PR)

// api.cu: per-thread error detail and launch count of the last call
void set_last_error(const char* msg);
void set_launch_count(int n);

}  // namespace spr
