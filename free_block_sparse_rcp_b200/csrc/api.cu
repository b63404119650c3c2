// C ABI of the SparsePR library: argument validation, workspace layout and the
// sequencing of the kernels of each call on the caller's stream.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace spr;

namespace {

thread_local char g_detail[512] = "no error";
thread_local int g_launches = 0;

sparsepr_status fail(sparsepr_status s, const char* msg) {
  snprintf(g_detail, sizeof(g_detail), "%s", msg);
  return s;
}

sparsepr_status failv(sparsepr_status s, const char* msg, long long v) {
  snprintf(g_detail, sizeof(g_detail), "%s (got %lld)", msg, v);
  return s;
}

sparsepr_status fail_cuda(cudaError_t e, const char* where) {
  snprintf(g_detail, sizeof(g_detail), "CUDA error in %s: %s", where, cudaGetErrorString(e));
  return SPARSEPR_ECUDA;
}

#define SPR_LAUNCH(expr)                                  \
  do {                                                    \
    cudaError_t e_ = (expr);                              \
    ++g_launches;                                         \
    if (e_ != cudaSuccess) return fail_cuda(e_, #expr);   \
  } while (0)
#define SPR_CUDA(expr)                                    \
  do {                                                    \
    cudaError_t e_ = (expr);                              \
    if (e_ != cudaSuccess) return fail_cuda(e_, #expr);   \
  } while (0)

constexpr size_t kSmemLimit = 227 * 1024;


size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
  // header
  size_t err;
  // partition
  size_t ident, sample_idx, metric, eigval, eigvec, proj, eig_lu, m_k, nu_k, key_init, C, m_q, nu_q, query_init, bias, wnorm,
      w_hi, w_lo, flag_count, flag_rows, corr_count, corr, slots, xnorm, mass, order, alpha;
  // attend
  size_t rlist, rcum, rcnt, tiles, tile_count;
  // frame-causal tables (zero-sized without frame ids): partition / attend / probe regions
  size_t c_fend, c_visk, c_qcum, a_visk, a_klist, a_tlim, p_fend;
  // probe
  size_t probe_grp, part_o, part_ml, o_sparse_p, lse_d, lse_s;
  size_t total;
  // forward extras
  size_t f_perm_q, f_perm_k, f_label_q, f_label_k, f_qoff, f_koff, f_route, f_bmask, f_rho, f_lse, f_probe_idx,
      f_probe_od, f_bfull, f_vr, f_w;
  size_t forward_total;
  int BH, max_tiles, T, S, DTk, DTq, F;
};

Layout make_layout(const sparsepr_params& p) {
  Layout L{};
  const size_t BH = (size_t)p.B * p.H, N = p.N, d = p.d;
  const size_t Gk = p.n_kgroups, Gq = p.n_qgroups, re = p.eig_rank, P = p.n_probes, r = p.sub_rank;
  L.BH = (int)BH;
  L.max_tiles = ceil_div(p.N, kAttnTileRows) + p.n_qgroups;
  L.T = ceil_div(p.N, p.block);
  L.S = probe_splits(p.N);
  // coordinate widths of the two k-means: response coordinates (r_e for keys, G_k for
  // queries), or the raw d-dimensional rows for the semantic-grouping baseline
  L.DTk = kmeans_dt(p.partition_mode == 1 ? p.d : p.eig_rank);
  L.DTq = kmeans_dt(p.partition_mode == 1 ? p.d : p.n_kgroups);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = al256(o + bytes); return at; };
  L.err = take(256);
  L.ident = take(p.partition_mode == 1 ? d * d * 4 : 0);
  L.sample_idx = take(BH * p.n_samples * 4);
  L.metric = take(BH * d * d * 4);
  L.eigval = take(BH * re * 4);
  L.eigvec = take(BH * d * re * 4);
  L.proj = take(BH * d * re * 4);
  L.eig_lu = take(BH * 3 * d * re * 4);
  const size_t GPmax = (size_t)kmeans_gp(p.n_kgroups > p.n_qgroups ? p.n_kgroups : p.n_qgroups);
  L.m_k = take(BH * Gk * d * 4);
  L.nu_k = take(BH * Gk * L.DTk * 4);
  L.key_init = take(BH * Gk * 4);
  L.C = take(BH * Gk * d * 4);
  L.m_q = take(BH * Gq * d * 4);
  L.nu_q = take(BH * Gq * L.DTq * 4);
  L.query_init = take(BH * Gq * 4);
  L.bias = take(BH * GPmax * 4);
  L.wnorm = take(BH * GPmax * 4);
  L.w_hi = take(BH * GPmax * d * 2);
  L.w_lo = take(BH * GPmax * d * 2 * 2);   // also holds the third part of C for the cell mass
  L.flag_count = take(BH * (size_t)kmeans_plan(1, p.N).SPH * 4);   // uncertified rows per k-means segment
  L.flag_rows = take(BH * N * 4);
  L.corr_count = take(BH * 4);
  L.corr = take(BH * N * 16);
  L.slots = take(kmeans_slots_bytes((int)BH, p.N, (int)GPmax, (int)d));
  L.xnorm = take(BH * N * 4);   // ||x||^2 of the rows of the running k-means
  L.mass = take(BH * Gq * Gk * 4);
  L.order = take(BH * Gq * Gk * 4);
  L.alpha = take(BH * 8);
  L.rlist = take(BH * Gq * Gk * 4);
  L.rcum = take(BH * Gq * (Gk + 1) * 4);
  L.rcnt = take(BH * Gq * 4);
  L.tiles = take(BH * L.max_tiles * 8);
  L.tile_count = take(BH * 4);
  L.F = p.frame_id ? p.n_frames : 0;
  {
    const size_t F = (size_t)L.F;
    L.c_fend = take(F * 4);
    L.c_visk = take(BH * Gk * F * 4);
    L.c_qcum = take(BH * Gq * F * 4);
    L.a_visk = take(BH * Gk * F * 4);
    L.a_klist = take(F ? BH * Gq * N * 4 : 0);
    L.a_tlim = take(BH * Gq * F * 4);
    L.p_fend = take(F * 4);
  }
  L.probe_grp = take(BH * P * 4);
  L.part_o = take(BH * L.S * 64 * 2 * d * 4);
  L.part_ml = take(BH * L.S * 64 * 4 * 4);
  L.o_sparse_p = take(BH * P * d * 4);
  L.lse_d = take(BH * P * 4);
  L.lse_s = take(BH * P * 4);
  L.total = o;
  L.f_perm_q = take(BH * N * 4);
  L.f_perm_k = take(BH * N * 4);
  L.f_label_q = take(BH * N * 4);
  L.f_label_k = take(BH * N * 4);
  L.f_qoff = take(BH * (Gq + 1) * 4);
  L.f_koff = take(BH * (Gk + 1) * 4);
  L.f_route = take(BH * Gq * Gk);
  L.f_bmask = take(BH * (size_t)L.T * L.T);
  L.f_rho = take(BH * 4);
  L.f_lse = take(BH * N * 4);
  L.f_probe_idx = take(BH * P * 4);
  L.f_probe_od = take(BH * P * d * 4);
  L.f_bfull = take(BH * d * 4);
  L.f_vr = take(BH * d * r * 4);
  L.f_w = take(BH * d * r * 4);
  L.forward_total = o;
  return L;
}

sparsepr_status check_params(const sparsepr_params* p) {
  if (!p) return fail(SPARSEPR_EINVAL, "params pointer is NULL");
  if (p->B < 1 || p->H < 1 || p->N < 1) return fail(SPARSEPR_EINVAL, "B, H and N must be >= 1");
  if ((long long)p->B * p->H * p->N > (1ll << 30)) return fail(SPARSEPR_EUNSUPPORTED, "B*H*N too large");
  if (p->d != 64 && p->d != 128) return failv(SPARSEPR_EUNSUPPORTED, "head dim d must be 64 or 128", p->d);
  if (p->block != 64 && p->block != 128) return failv(SPARSEPR_EINVAL, "block must be 64 or 128", p->block);
  if (!(p->density > 0.f) || !(p->density <= 1.f)) return fail(SPARSEPR_EINVAL, "density must be in (0, 1]");
  const int gmax = p->N < 1024 ? p->N : 1024;
  if (p->n_kgroups < 1 || p->n_kgroups > gmax) return failv(SPARSEPR_EINVAL, "n_kgroups must be in [1, min(N,1024)]", p->n_kgroups);
  if (p->n_qgroups < 1 || p->n_qgroups > gmax) return failv(SPARSEPR_EINVAL, "n_qgroups must be in [1, min(N,1024)]", p->n_qgroups);
  if (p->n_samples < 1 || p->n_samples > gmax) return failv(SPARSEPR_EINVAL, "n_samples must be in [1, min(N,1024)]", p->n_samples);
  const int pmax = p->N < 64 ? p->N : 64;
  if (p->n_probes < 1 || p->n_probes > pmax) return failv(SPARSEPR_EINVAL, "n_probes must be in [1, min(N,64)]", p->n_probes);
  if (p->eig_rank < 1 || p->eig_rank > p->d) return failv(SPARSEPR_EINVAL, "eig_rank must be in [1, d]", p->eig_rank);
  if (p->eig_rank > 64 || metric_eigen_smem(p->d, p->eig_rank) > kSmemLimit)
    return failv(SPARSEPR_EUNSUPPORTED, "eig_rank > 64 not built (single-CTA eigensolver)", p->eig_rank);
  if (p->sub_rank < 1 || p->sub_rank > p->n_probes || p->sub_rank > p->d)
    return failv(SPARSEPR_EINVAL, "sub_rank must be in [1, min(d, n_probes)]", p->sub_rank);
  if (p->kmeans_iters < 1 || p->kmeans_iters > 64) return failv(SPARSEPR_EINVAL, "kmeans_iters must be in [1, 64]", p->kmeans_iters);
  if (!(p->ridge_lambda > 0.f) || !isfinite(p->ridge_lambda)) return fail(SPARSEPR_EINVAL, "ridge_lambda must be > 0");
  if (!(p->scale >= 0.f) || !isfinite(p->scale)) return fail(SPARSEPR_EINVAL, "scale must be >= 0");
  if (p->fit_weighted != 0 && p->fit_weighted != 1)
    return failv(SPARSEPR_EINVAL, "fit_weighted must be 0 or 1", p->fit_weighted);
  if (p->fit_input != 0 && p->fit_input != 1)
    return failv(SPARSEPR_EINVAL, "fit_input must be 0 (whole sparse output) or 1 (projected on the subspace)",
                 p->fit_input);
  if (p->head_offset < 0) return failv(SPARSEPR_EINVAL, "head_offset must be >= 0", p->head_offset);
  if (p->heads_total != 0 && (p->heads_total < 0 || (long long)p->heads_total < (long long)p->head_offset + p->H))
    return failv(SPARSEPR_EINVAL, "heads_total must be 0 or >= head_offset + H", p->heads_total);
  if ((long long)(p->B - 1) * (p->heads_total ? p->heads_total : p->H) + p->head_offset + p->H > (1ll << 28))
    return fail(SPARSEPR_EINVAL, "layer head index out of range");
  if (p->partition_mode != 0 && p->partition_mode != 1)
    return failv(SPARSEPR_EINVAL, "partition_mode must be 0 (response-coupled) or 1 (semantic)", p->partition_mode);
  if (p->frame_id) {
    if (p->n_frames < 1 || p->n_frames > kMaxFrames)
      return failv(SPARSEPR_EINVAL, "n_frames must be in [1, 64] with frame_id", p->n_frames);
    if (p->N > 65535) return failv(SPARSEPR_EUNSUPPORTED, "frame-causal calls need N <= 65535", p->N);
    if (causal_stream_smem(p->n_kgroups, p->n_frames) > kSmemLimit)
      return fail(SPARSEPR_EUNSUPPORTED, "too many K/V groups x frames for the causal key stream");
  }
  if (p->density < 1.f &&
      (double)p->density * (double)p->N * (double)p->N < (double)p->n_probes * (double)p->N)
    return fail(SPARSEPR_EINVAL, "density is below the probe floor n_probes/N");
  // kernel limits
  if (p->n_kgroups > 128) return fail(SPARSEPR_EUNSUPPORTED, "n_kgroups > 128 (query coordinates wider than 128) not built");
  if (p->n_qgroups > 128) return fail(SPARSEPR_EUNSUPPORTED, "n_qgroups > 128 not built");
  const int Dk = p->partition_mode == 1 ? p->d : p->eig_rank, Dq = p->partition_mode == 1 ? p->d : p->n_kgroups;
  if (recheck_smem(p->d, Dq, kmeans_dt(Dq), p->n_qgroups, p->N) > kSmemLimit ||
      recheck_smem(p->d, Dk, kmeans_dt(Dk), p->n_kgroups, p->N) > kSmemLimit ||
      centroid_weights_smem(p->d, Dq > Dk ? Dq : Dk, p->N) > kSmemLimit ||
      assign_acc_smem(p->d, kmeans_gp(p->n_kgroups > p->n_qgroups ? p->n_kgroups : p->n_qgroups)) > kSmemLimit)
    return fail(SPARSEPR_EUNSUPPORTED, "too many groups for the k-means kernels");
  if (route_select_smem(p->n_qgroups, p->n_kgroups) > kSmemLimit)
    return fail(SPARSEPR_EUNSUPPORTED, "too many groups for the route selection kernel");
  if (cell_mass_tc_smem(p->d, kmeans_gp(p->n_kgroups), p->frame_id ? p->n_frames : 0) > kSmemLimit)
    return fail(SPARSEPR_EUNSUPPORTED, "too many K/V groups for the cell-mass kernel");
  if ((size_t)p->d * p->sub_rank > 64 * 65 || probe_fit_smem(p->d, p->sub_rank) > kSmemLimit)
    return failv(SPARSEPR_EUNSUPPORTED, "sub_rank too large for the single-CTA fit (d*r)", (long long)p->d * p->sub_rank);
  if (attn_tc_smem_bytes(p->d, p->n_kgroups) > kSmemLimit || probe_tc_smem_bytes(p->d, p->n_kgroups) > kSmemLimit)
    return fail(SPARSEPR_EUNSUPPORTED, "too many K/V groups for the attention kernels");
  return SPARSEPR_OK;
}

sparsepr_status check_ws(const sparsepr_params* p, void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(SPARSEPR_EINVAL, "workspace is NULL");
  if (((uintptr_t)ws & 255) != 0) return fail(SPARSEPR_EWORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return failv(SPARSEPR_EWORKSPACE, "workspace too small (bytes needed)", (long long)need);
  (void)p;
  return SPARSEPR_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

float eff_scale(const sparsepr_params& p) { return p.scale > 0.f ? p.scale : 1.0f / sqrtf((float)p.d); }

// layer-wide head index of the random streams (head_offset / heads_total)
HeadMap head_map(const sparsepr_params& p) {
  HeadMap hm;
  hm.H = p.H;
  hm.total = p.heads_total ? p.heads_total : p.H;
  hm.offset = p.head_offset;
  return hm;
}

#define SPR_CHECK(expr)                          \
  do {                                           \
    sparsepr_status s_ = (expr);                 \
    if (s_ != SPARSEPR_OK) return s_;            \
  } while (0)
#define SPR_NONNULL(ptr)                                                                  \
  do {                                                                                    \
    if (!(ptr)) return fail(SPARSEPR_EINVAL, "required pointer " #ptr " is NULL");        \
  } while (0)
// bf16 token tensors are read and written by TMA: non-NULL and 16-byte aligned
#define SPR_TILED(ptr)                                                                    \
  do {                                                                                    \
    SPR_NONNULL(ptr);                                                                     \
    if ((uintptr_t)(ptr) & 15u) return fail(SPARSEPR_EINVAL, "tensor " #ptr " is not 16-byte aligned"); \
  } while (0)

// ---------------------------------------------------------------------------
sparsepr_status run_partition(const sparsepr_params& p, const Layout& L, const void* Q, const void* K, int* perm_q,
                              int* perm_k, int* label_q, int* label_k, int* qoff, int* koff, unsigned char* route,
                              unsigned char* bmask, float* rho, const sparsepr_partition_trace* tr, void* ws,
                              cudaStream_t st, bool clear_err = true) {
  const int BH = L.BH, N = p.N, d = p.d, Gk = p.n_kgroups, Gq = p.n_qgroups, re = p.eig_rank;
  const float scale = eff_scale(p);
  int* err = at<int>(ws, L.err);
  if (clear_err) SPR_CUDA(cudaMemsetAsync(err, 0, 4, st));
  float* metric = at<float>(ws, L.metric);
  float* proj = at<float>(ws, L.proj);
  const bool semantic = p.partition_mode == 1;
  if (!semantic) {
    SPR_LAUNCH(launch_sample_metric(Q, BH, N, d, p.n_samples, p.seed, head_map(p), metric, at<int>(ws, L.sample_idx),
                                    err, st));
    SPR_LAUNCH(launch_metric_eigen(metric, BH, d, re, at<float>(ws, L.eigval), at<float>(ws, L.eigvec), proj,
                                   at<float>(ws, L.eig_lu), st));
    if (tr && tr->key_coords) SPR_LAUNCH(launch_key_coords(K, BH, N, d, re, proj, tr->key_coords, st));
  } else {
    SPR_LAUNCH(launch_identity(at<float>(ws, L.ident), d, st));
  }
  float* bias = at<float>(ws, L.bias);
  float* wnorm = at<float>(ws, L.wnorm);
  void* w_hi = at<char>(ws, L.w_hi);
  void* w_lo = at<char>(ws, L.w_lo);
  int* fcount = at<int>(ws, L.flag_count);
  int* frows = at<int>(ws, L.flag_rows);
  int* ccount = at<int>(ws, L.corr_count);
  void* corr = at<char>(ws, L.corr);
  void* slots = at<char>(ws, L.slots);
  // One Lloyd k-means of the rows X (bf16, d) on coordinates A x; A(j, c) = a_scale * A[j*sj + c*sc].
  // Each pass assigns every row and leaves the per-group sums of its rows for the next
  // centroid update; means_out (if set) receives the means of the final groups.
  auto kmeans = [&](const void* X, int G, int purpose, const float* A, size_t a_head, int sj, int sc, float a_scale,
                    int D, int DT, float* m, float* nu, int* init, int* labels, int* perm, int* off,
                    int* trace_iters, float* means_out) -> sparsepr_status {
    SPR_LAUNCH(launch_seed_rows(X, BH, N, d, G, p.seed, head_map(p), purpose, m, init, err, st));
    for (int t = 0; t < p.kmeans_iters; ++t) {
      int* trc = trace_iters ? trace_iters + (size_t)t * BH * N : nullptr;
      SPR_LAUNCH(launch_centroid_weights(m, BH, G, d, A, a_head, sj, sc, a_scale, D, DT, t == 0 ? 0 : 1, slots,
                                         ccount, corr, X, N, nu, bias, wnorm, w_hi, w_lo, err, st));
      SPR_CUDA(cudaMemsetAsync(ccount, 0, (size_t)BH * 4, st));
      SPR_LAUNCH(launch_assign_acc(X, BH, N, d, G, w_hi, w_lo, bias, wnorm, labels, trc, fcount, frows, slots,
                                   at<float>(ws, L.xnorm), t == 0 ? 1 : 0, err, st));
      SPR_LAUNCH(launch_assign_recheck(X, BH, N, d, A, a_head, sj, sc, a_scale, D, nu, G, fcount, frows, labels,
                                       trc, ccount, corr, st));
    }
    SPR_LAUNCH(launch_group_sort(labels, BH, N, G, perm, off, err, st));
    if (means_out)
      SPR_LAUNCH(launch_centroid_weights(means_out, BH, G, d, A, a_head, sj, sc, a_scale, D, DT, 2, slots, ccount,
                                         corr, X, N, nullptr, nullptr, nullptr, nullptr, nullptr, err, st));
    return SPARSEPR_OK;
  };
  // keys on y = Lambda^{1/2} U^T k: A(j, c) = proj[c][j]; K/V group centroids = mean raw key
  // of the final groups (empty group -> 0)
  float* C = at<float>(ws, L.C);
  const float* ident = at<float>(ws, L.ident);
  if (!semantic) {
    SPR_CHECK(kmeans(K, Gk, PURPOSE_KEY_KMEANS, proj, (size_t)d * re, 1, re, 1.0f, re, L.DTk, at<float>(ws, L.m_k),
                     at<float>(ws, L.nu_k), at<int>(ws, L.key_init), label_k, perm_k, koff,
                     tr ? tr->key_label_iters : nullptr, C));
  } else {
    // semantic-grouping baseline: keys clustered on their raw rows (A = identity)
    SPR_CHECK(kmeans(K, Gk, PURPOSE_KEY_KMEANS, ident, 0, d, 1, 1.0f, d, L.DTk, at<float>(ws, L.m_k),
                     at<float>(ws, L.nu_k), at<int>(ws, L.key_init), label_k, perm_k, koff,
                     tr ? tr->key_label_iters : nullptr, C));
  }
  if (tr && tr->query_coords) SPR_LAUNCH(launch_query_coords(Q, BH, N, d, C, Gk, scale, tr->query_coords, st));
  // queries on z = s C q: A(j, c) = s * C[j][c]  (semantic baseline: on the raw rows)
  if (!semantic)
    SPR_CHECK(kmeans(Q, Gq, PURPOSE_QUERY_KMEANS, C, (size_t)Gk * d, d, 1, scale, Gk, L.DTq, at<float>(ws, L.m_q),
                     at<float>(ws, L.nu_q), at<int>(ws, L.query_init), label_q, perm_q, qoff,
                     tr ? tr->query_label_iters : nullptr, nullptr));
  else
    SPR_CHECK(kmeans(Q, Gq, PURPOSE_QUERY_KMEANS, ident, 0, d, 1, 1.0f, d, L.DTq, at<float>(ws, L.m_q),
                     at<float>(ws, L.nu_q), at<int>(ws, L.query_init), label_q, perm_q, qoff,
                     tr ? tr->query_label_iters : nullptr, nullptr));
  float* mass = at<float>(ws, L.mass);
  // frame-causal: visible keys per (K/V group, frame), query frame histograms, frame ends
  Causal cz{};
  if (p.frame_id) {
    cz.frame_id = p.frame_id;
    cz.F = L.F;
    cz.fend = at<int>(ws, L.c_fend);
    cz.visk = at<int>(ws, L.c_visk);
    cz.qcum = at<int>(ws, L.c_qcum);
    SPR_LAUNCH(launch_frame_ends(p.frame_id, N, L.F, at<int>(ws, L.c_fend), err, st));
    SPR_LAUNCH(launch_group_frame_cum(perm_k, koff, p.frame_id, BH, N, Gk, L.F, at<int>(ws, L.c_visk), err, st));
    SPR_LAUNCH(launch_group_frame_cum(perm_q, qoff, p.frame_id, BH, N, Gq, L.F, at<int>(ws, L.c_qcum), err, st));
  }
  // the weight buffers are free again: they hold the three bf16 parts of C
  const size_t cpart = (size_t)BH * kmeans_gp(Gk) * d * 2;
  SPR_LAUNCH(launch_cell_mass_tc(Q, BH, N, d, Gq, Gk, perm_q, qoff, koff, C, scale, w_hi, w_lo,
                                 at<char>(ws, L.w_lo) + cpart, cz, mass, err, st));
  ++g_launches;   // the cell-mass launcher also splits C into its bf16 parts (a second kernel)
  SPR_LAUNCH(launch_route_select(mass, BH, N, Gq, Gk, qoff, koff, p.density, p.n_probes, cz, at<int>(ws, L.order),
                                 route, rho, at<double>(ws, L.alpha), st));
  if (bmask)
    SPR_LAUNCH(launch_block_mask(route, BH, N, Gq, Gk, p.block, perm_q, label_q, perm_k, label_k, bmask, st));
  if (tr) {
    auto cp = [&](void* dst, size_t off, size_t bytes) -> cudaError_t {
      return dst ? cudaMemcpyAsync(dst, at<char>(ws, off), bytes, cudaMemcpyDeviceToDevice, st) : cudaSuccess;
    };
    const size_t bh = BH;
    if (!semantic) {
      SPR_CUDA(cp(tr->sample_idx, L.sample_idx, bh * p.n_samples * 4));
      SPR_CUDA(cp(tr->metric, L.metric, bh * d * d * 4));
      SPR_CUDA(cp(tr->eigval, L.eigval, bh * re * 4));
      SPR_CUDA(cp(tr->eigvec, L.eigvec, bh * d * re * 4));
    }
    SPR_CUDA(cp(tr->key_init, L.key_init, bh * Gk * 4));
    SPR_CUDA(cp(tr->key_centroids, L.C, bh * Gk * d * 4));
    SPR_CUDA(cp(tr->query_init, L.query_init, bh * Gq * 4));
    SPR_CUDA(cp(tr->cell_mass, L.mass, bh * Gq * Gk * 4));
    SPR_CUDA(cp(tr->alpha, L.alpha, bh * 8));
  }
  return SPARSEPR_OK;
}

sparsepr_status run_attend(const sparsepr_params& p, const Layout& L, const void* Q, const void* K, const void* V,
                           const int* perm_q, const int* perm_k, const int* qoff, const int* koff,
                           const unsigned char* route, void* O, float* lse, void* ws, cudaStream_t st) {
  int* rlist = at<int>(ws, L.rlist);
  int* rcum = at<int>(ws, L.rcum);
  int* rcnt = at<int>(ws, L.rcnt);
  int2* tiles = at<int2>(ws, L.tiles);
  int* tcount = at<int>(ws, L.tile_count);
  SPR_LAUNCH(launch_worklist(route, qoff, koff, L.BH, p.n_qgroups, p.n_kgroups, kAttnTileRows, L.max_tiles, rlist,
                             rcum, rcnt, tiles, tcount, st));
  AttnArgs a{};
  a.Q = Q; a.K = K; a.V = V;
  a.BH = L.BH; a.N = p.N; a.D = p.d; a.Gq = p.n_qgroups; a.Gk = p.n_kgroups;
  a.perm_q = perm_q; a.perm_k = perm_k; a.qoff = qoff; a.koff = koff;
  a.rlist = rlist; a.rcum = rcum; a.rcnt = rcnt; a.tiles = tiles; a.tile_count = tcount;
  a.max_tiles = L.max_tiles;
  a.scale_log2 = eff_scale(p) * 1.4426950408889634f;
  a.O = O; a.lse = lse; a.err = at<int>(ws, L.err);
  if (p.frame_id) {
    // each query group's routed keys in frame-major order, and its prefix per frame
    int* visk = at<int>(ws, L.a_visk);
    SPR_LAUNCH(launch_group_frame_cum(perm_k, koff, p.frame_id, L.BH, p.N, p.n_kgroups, L.F, visk, a.err, st));
    SPR_LAUNCH(launch_causal_stream(rlist, rcnt, koff, perm_k, visk, L.BH, p.N, p.n_qgroups, p.n_kgroups, L.F,
                                    at<int>(ws, L.a_klist), at<int>(ws, L.a_tlim), a.err, st));
    a.cz.frame_id = p.frame_id;
    a.cz.F = L.F;
    a.cz.klist = at<int>(ws, L.a_klist);
    a.cz.tlim = at<int>(ws, L.a_tlim);
  }
  SPR_LAUNCH(launch_attention_tc(a, false, st));
  return SPARSEPR_OK;
}

sparsepr_status run_probe_fit(const sparsepr_params& p, const Layout& L, const void* Q, const void* K,
                              const void* V, const int* label_k, const int* perm_q, const int* qoff,
                              const unsigned char* route, int* probe_idx, float* probe_od, float* bfull,
                              float* Vr, float* W, float* Bmat, const sparsepr_probe_trace* tr, void* ws,
                              cudaStream_t st) {
  const int BH = L.BH, N = p.N, d = p.d, P = p.n_probes;
  int* pgrp = at<int>(ws, L.probe_grp);
  SPR_LAUNCH(launch_probe_pick(perm_q, qoff, BH, N, p.n_qgroups, P, p.seed, head_map(p), probe_idx, pgrp,
                               at<int>(ws, L.err), st));
  float* part_o = at<float>(ws, L.part_o);
  float* part_ml = at<float>(ws, L.part_ml);
  Causal cz{};
  if (p.frame_id) {
    cz.frame_id = p.frame_id;
    cz.F = L.F;
    cz.fend = at<int>(ws, L.p_fend);
    SPR_LAUNCH(launch_frame_ends(p.frame_id, N, L.F, at<int>(ws, L.p_fend), at<int>(ws, L.err), st));
  }
  SPR_LAUNCH(launch_probe_attn(Q, K, V, BH, N, d, p.n_kgroups, p.n_qgroups, P, probe_idx, pgrp, label_k, route,
                               eff_scale(p) * 1.4426950408889634f, cz, part_o, part_ml, at<int>(ws, L.err), st));
  float* osp = at<float>(ws, L.o_sparse_p);
  float* lsd = at<float>(ws, L.lse_d);
  float* lss = at<float>(ws, L.lse_s);
  SPR_LAUNCH(launch_probe_combine(part_o, part_ml, BH, N, P, d, probe_od, osp, lsd, lss, st));
  SPR_LAUNCH(launch_probe_fit(probe_od, osp, BH, d, P, p.sub_rank, (double)p.ridge_lambda, Vr, W, bfull, Bmat,
                              tr ? tr->sigma : nullptr, tr ? tr->b_sub : nullptr, p.fit_weighted ? pgrp : nullptr,
                              qoff, p.n_qgroups, p.fit_input == 0, st));
  if (tr) {
    if (tr->probe_o_sparse)
      SPR_CUDA(cudaMemcpyAsync(tr->probe_o_sparse, osp, (size_t)BH * P * d * 4, cudaMemcpyDeviceToDevice, st));
    if (tr->probe_lse_dense)
      SPR_CUDA(cudaMemcpyAsync(tr->probe_lse_dense, lsd, (size_t)BH * P * 4, cudaMemcpyDeviceToDevice, st));
    if (tr->probe_lse_sparse)
      SPR_CUDA(cudaMemcpyAsync(tr->probe_lse_sparse, lss, (size_t)BH * P * 4, cudaMemcpyDeviceToDevice, st));
  }
  return SPARSEPR_OK;
}

sparsepr_status run_reconstruct(const sparsepr_params& p, int BH, const void* Os, const int* probe_idx,
                                const float* probe_od, const float* bfull, const float* Vr, const float* W, void* O,
                                cudaStream_t st) {
  SPR_LAUNCH(launch_reconstruct(Os, BH, p.N, p.d, p.sub_rank, W, Vr, bfull, O, st));
  SPR_LAUNCH(launch_probe_scatter(probe_idx, probe_od, BH, p.N, p.n_probes, p.d, O, st));
  return SPARSEPR_OK;
}

}  // namespace

namespace spr {
void set_last_error(const char* msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg); }
void set_launch_count(int n) { g_launches = n; }
}  // namespace spr

// ===========================================================================
extern "C" {

size_t sparsepr_workspace_bytes(const sparsepr_params* p) {
  if (check_params(p) != SPARSEPR_OK) return 0;
  return make_layout(*p).total;
}

size_t sparsepr_forward_workspace_bytes(const sparsepr_params* p) {
  if (check_params(p) != SPARSEPR_OK) return 0;
  return make_layout(*p).forward_total;
}

sparsepr_status sparsepr_validate(const sparsepr_params* p) { return check_params(p); }

sparsepr_status sparsepr_partition(const sparsepr_params* p, const void* Q, const void* K, int* perm_q, int* perm_k,
                                   int* label_q, int* label_k, int* qoff, int* koff, unsigned char* route,
                                   unsigned char* block_mask, float* rho_exec, const sparsepr_partition_trace* trace,
                                   void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_TILED(Q); SPR_TILED(K); SPR_NONNULL(perm_q); SPR_NONNULL(perm_k); SPR_NONNULL(label_q);
  SPR_NONNULL(label_k); SPR_NONNULL(qoff); SPR_NONNULL(koff); SPR_NONNULL(route); SPR_NONNULL(rho_exec);
  const Layout L = make_layout(*p);
  SPR_CHECK(check_ws(p, workspace, ws_bytes, L.total));
  return run_partition(*p, L, Q, K, perm_q, perm_k, label_q, label_k, qoff, koff, route, block_mask, rho_exec,
                       trace, workspace, (cudaStream_t)stream);
}

sparsepr_status sparsepr_attend(const sparsepr_params* p, const void* Q, const void* K, const void* V,
                                const int* perm_q, const int* perm_k, const int* qoff, const int* koff,
                                const unsigned char* route, void* O_sparse, float* lse, void* workspace,
                                size_t ws_bytes, void* stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_TILED(Q); SPR_TILED(K); SPR_TILED(V); SPR_NONNULL(perm_q); SPR_NONNULL(perm_k); SPR_NONNULL(qoff);
  SPR_NONNULL(koff); SPR_NONNULL(route); SPR_TILED(O_sparse);
  const Layout L = make_layout(*p);
  SPR_CHECK(check_ws(p, workspace, ws_bytes, L.total));
  return run_attend(*p, L, Q, K, V, perm_q, perm_k, qoff, koff, route, O_sparse, lse, workspace,
                    (cudaStream_t)stream);
}

sparsepr_status sparsepr_probe_fit(const sparsepr_params* p, const void* Q, const void* K, const void* V,
                                   const int* label_k, const int* perm_q, const int* qoff, const unsigned char* route,
                                   int* probe_idx, float* probe_o_dense, float* b_full, float* Vr, float* W,
                                   float* Bmat, const sparsepr_probe_trace* trace, void* workspace, size_t ws_bytes,
                                   void* stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_TILED(Q); SPR_TILED(K); SPR_TILED(V); SPR_NONNULL(label_k); SPR_NONNULL(perm_q); SPR_NONNULL(qoff);
  SPR_NONNULL(route); SPR_NONNULL(probe_idx); SPR_NONNULL(probe_o_dense); SPR_NONNULL(b_full); SPR_NONNULL(Vr);
  SPR_NONNULL(W);
  const Layout L = make_layout(*p);
  SPR_CHECK(check_ws(p, workspace, ws_bytes, L.total));
  return run_probe_fit(*p, L, Q, K, V, label_k, perm_q, qoff, route, probe_idx, probe_o_dense, b_full, Vr, W, Bmat,
                       trace, workspace, (cudaStream_t)stream);
}

sparsepr_status sparsepr_reconstruct(const sparsepr_params* p, const void* O_sparse, const int* probe_idx,
                                     const float* probe_o_dense, const float* b_full, const float* Vr,
                                     const float* W, void* O, void* stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_TILED(O_sparse); SPR_NONNULL(probe_idx); SPR_NONNULL(probe_o_dense); SPR_NONNULL(b_full); SPR_NONNULL(Vr);
  SPR_NONNULL(W); SPR_TILED(O);
  return run_reconstruct(*p, p->B * p->H, O_sparse, probe_idx, probe_o_dense, b_full, Vr, W, O,
                         (cudaStream_t)stream);
}

// A second stream forked from `st` for the duration of one call: side() is a fresh
// non-blocking stream of the highest priority that starts after the work already on `st`
// (or `st` itself if a stream or event cannot be created, or if `st` is being captured
// into a CUDA graph, where a stream created and destroyed inside the capture has no
// place); join() makes `st` wait for it.  The stream and events are released when the
// object goes out of scope (the driver frees them once their work completes).
class ForkJoin {
 public:
  explicit ForkJoin(cudaStream_t st) : st_(st) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st_, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
      cudaGetLastError();
      return;
    }
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) hi = 0;
    if (cudaStreamCreateWithPriority(&side_, cudaStreamNonBlocking, hi) != cudaSuccess) { side_ = nullptr; return; }
    if (cudaEventCreateWithFlags(&fork_, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&done_, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventRecord(fork_, st_) != cudaSuccess || cudaStreamWaitEvent(side_, fork_, 0) != cudaSuccess) {
      release();
      cudaGetLastError();
    }
  }
  // on an early return the caller's stream still waits for whatever the side stream took
  ~ForkJoin() {
    if (side_ && !joined_ && cudaEventRecord(done_, side_) == cudaSuccess) cudaStreamWaitEvent(st_, done_, 0);
    release();
  }
  cudaStream_t side() const { return side_ ? side_ : st_; }
  void mark_side_done() {
    if (side_ && cudaEventRecord(done_, side_) != cudaSuccess) failed_ = true;
  }
  sparsepr_status join() {
    if (!side_) return SPARSEPR_OK;
    if (failed_) return fail(SPARSEPR_ECUDA, "cudaEventRecord on the probe stream failed");
    const cudaError_t e = cudaStreamWaitEvent(st_, done_, 0);
    joined_ = e == cudaSuccess;
    return joined_ ? SPARSEPR_OK : fail_cuda(e, "cudaStreamWaitEvent(stream, probe path done)");
  }

 private:
  void release() {
    if (fork_) cudaEventDestroy(fork_);
    if (done_) cudaEventDestroy(done_);
    if (side_) cudaStreamDestroy(side_);
    fork_ = done_ = nullptr;
    side_ = nullptr;
  }
  cudaStream_t st_;
  cudaStream_t side_ = nullptr;
  cudaEvent_t fork_ = nullptr, done_ = nullptr;
  bool failed_ = false, joined_ = false;
};

// The whole call on device buffers; clear_err: reset the workspace error word first.
static sparsepr_status forward_impl(const sparsepr_params* p, const void* Q, const void* K, const void* V, void* O,
                             float* rho_exec, void* workspace, size_t ws_bytes, void* stream, bool clear_err) {
  SPR_CHECK(check_params(p));
  SPR_TILED(Q); SPR_TILED(K); SPR_TILED(V); SPR_TILED(O);
  const Layout L = make_layout(*p);
  SPR_CHECK(check_ws(p, workspace, ws_bytes, L.forward_total));
  cudaStream_t st = (cudaStream_t)stream;
  void* ws = workspace;
  int* perm_q = at<int>(ws, L.f_perm_q);
  int* perm_k = at<int>(ws, L.f_perm_k);
  int* label_q = at<int>(ws, L.f_label_q);
  int* label_k = at<int>(ws, L.f_label_k);
  int* qoff = at<int>(ws, L.f_qoff);
  int* koff = at<int>(ws, L.f_koff);
  unsigned char* route = at<unsigned char>(ws, L.f_route);
  float* rho = rho_exec ? rho_exec : at<float>(ws, L.f_rho);
  SPR_CHECK(run_partition(*p, L, Q, K, perm_q, perm_k, label_q, label_k, qoff, koff, route, nullptr, rho, nullptr,
                          ws, st, clear_err));
  int* pidx = at<int>(ws, L.f_probe_idx);
  float* pod = at<float>(ws, L.f_probe_od);
  float* bfull = at<float>(ws, L.f_bfull);
  float* vr = at<float>(ws, L.f_vr);
  float* w = at<float>(ws, L.f_w);
  // attend and probe_fit read only the partition and write disjoint workspace regions: the
  // probe path runs on a higher-priority stream of this call beside the routed attention and
  // joins before the correction (one stream for both if the second cannot be created)
  ForkJoin fj(st);
  SPR_CHECK(run_probe_fit(*p, L, Q, K, V, label_k, perm_q, qoff, route, pidx, pod, bfull, vr, w, nullptr, nullptr,
                          ws, fj.side()));
  fj.mark_side_done();
  SPR_CHECK(run_attend(*p, L, Q, K, V, perm_q, perm_k, qoff, koff, route, O, at<float>(ws, L.f_lse), ws, st));
  SPR_CHECK(fj.join());
  SPR_CHECK(run_reconstruct(*p, L.BH, O, pidx, pod, bfull, vr, w, O, st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_forward(const sparsepr_params* p, const void* Q, const void* K, const void* V, void* O,
                                 float* rho_exec, void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  return forward_impl(p, Q, K, V, O, rho_exec, workspace, ws_bytes, stream, true);
}

sparsepr_status sparsepr_forward_host(const sparsepr_params* p, const void* Q_host, const void* K_host,
                                      const void* V_host, void* O_host, void* qkv_dev, void* o_dev, void* workspace,
                                      size_t ws_bytes, void* stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_NONNULL(Q_host); SPR_NONNULL(K_host); SPR_NONNULL(V_host); SPR_NONNULL(O_host); SPR_TILED(qkv_dev);
  SPR_TILED(o_dev);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t bytes = (size_t)p->B * p->H * p->N * p->d * 2;
  char* q = static_cast<char*>(qkv_dev);
  SPR_CUDA(cudaMemcpyAsync(q, Q_host, bytes, cudaMemcpyHostToDevice, st));
  SPR_CUDA(cudaMemcpyAsync(q + bytes, K_host, bytes, cudaMemcpyHostToDevice, st));
  SPR_CUDA(cudaMemcpyAsync(q + 2 * bytes, V_host, bytes, cudaMemcpyHostToDevice, st));
  SPR_CHECK(sparsepr_forward(p, q, q + bytes, q + 2 * bytes, o_dev, nullptr, workspace, ws_bytes, stream));
  SPR_CUDA(cudaMemcpyAsync(O_host, o_dev, bytes, cudaMemcpyDeviceToHost, st));
  return SPARSEPR_OK;
}

sparsepr_status sparsepr_forward_host_chunked(const sparsepr_params* p, const void* Q_host, const void* K_host,
                                              const void* V_host, void* O_host, void* qkv_dev, void* o_dev,
                                              int n_chunks, void* workspace, size_t ws_bytes, void* stream,
                                              void* copy_in_stream, void* copy_out_stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_NONNULL(Q_host); SPR_NONNULL(K_host); SPR_NONNULL(V_host); SPR_NONNULL(O_host); SPR_TILED(qkv_dev);
  SPR_TILED(o_dev);
  const int BH = p->B * p->H;
  if (n_chunks < 1 || n_chunks > BH) return failv(SPARSEPR_EINVAL, "n_chunks must be in [1, B*H]", n_chunks);
  // chunk ranges over the flattened heads; when the layer numbering is not the identity a
  // chunk may not cross a batch element (each chunk is a B = 1 call over consecutive layer heads)
  const HeadMap hm = head_map(*p);
  const bool ident = hm.total == p->H && hm.offset == 0;
  const int per = ceil_div(BH, n_chunks);
  constexpr int kMaxChunks = 512;
  int starts[kMaxChunks + 1];
  int nc = 0;
  for (int h0 = 0; h0 < BH;) {
    int h1 = h0 + per < BH ? h0 + per : BH;
    if (!ident && (h0 / p->H) != ((h1 - 1) / p->H)) h1 = (h0 / p->H + 1) * p->H;
    if (nc >= kMaxChunks) return fail(SPARSEPR_EUNSUPPORTED, "more than 512 chunks");
    starts[nc++] = h0;
    h0 = h1;
  }
  starts[nc] = BH;
  int hmax = 0;
  for (int c = 0; c < nc; ++c) hmax = starts[c + 1] - starts[c] > hmax ? starts[c + 1] - starts[c] : hmax;
  sparsepr_params pc = *p;
  pc.B = 1;
  pc.H = hmax;
  pc.head_offset = 0;
  pc.heads_total = 0;
  SPR_CHECK(check_params(&pc));
  SPR_CHECK(check_ws(&pc, workspace, ws_bytes, make_layout(pc).forward_total));
  cudaStream_t st = (cudaStream_t)stream;
  cudaStream_t sin = copy_in_stream ? (cudaStream_t)copy_in_stream : st;
  cudaStream_t sout = copy_out_stream ? (cudaStream_t)copy_out_stream : st;
  const size_t head_bytes = (size_t)p->N * p->d * 2, bytes = (size_t)BH * head_bytes;
  // events are created here and released once enqueued (a pending event is freed when it
  // completes); none outlives the call
  cudaEvent_t ev[2 * kMaxChunks + 2];
  const int nev = 2 * nc + 2;
  int made = 0;
  sparsepr_status status = SPARSEPR_OK;
  auto cuda = [&](cudaError_t e, const char* where) -> bool {
    if (e != cudaSuccess && status == SPARSEPR_OK) status = fail_cuda(e, where);
    return e == cudaSuccess;
  };
  for (; made < nev; ++made)
    if (!cuda(cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming), "cudaEventCreateWithFlags")) break;
  if (status == SPARSEPR_OK) {
    cudaEvent_t e_start = ev[0], e_end = ev[1];
    char* q = static_cast<char*>(qkv_dev);
    char* o = static_cast<char*>(o_dev);
    // the copies in wait for earlier work on `stream` (which may still read the staging buffers)
    // the copies in wait for earlier work on `stream` (which may still read the staging
    // buffers); the error word is cleared once, so a device error of any chunk stays visible
    bool ok = cuda(cudaMemsetAsync(workspace, 0, 4, st), "cudaMemsetAsync") &&
              cuda(cudaEventRecord(e_start, st), "cudaEventRecord") &&
              cuda(cudaStreamWaitEvent(sin, e_start, 0), "cudaStreamWaitEvent");
    int launches = 0;
    for (int c = 0; ok && c < nc; ++c) {
      const int h0 = starts[c], h1 = starts[c + 1];
      const size_t off = (size_t)h0 * head_bytes, len = (size_t)(h1 - h0) * head_bytes;
      cudaEvent_t e_in = ev[2 + 2 * c], e_done = ev[3 + 2 * c];
      ok = cuda(cudaMemcpyAsync(q + off, static_cast<const char*>(Q_host) + off, len, cudaMemcpyHostToDevice, sin),
                "cudaMemcpyAsync Q") &&
           cuda(cudaMemcpyAsync(q + bytes + off, static_cast<const char*>(K_host) + off, len,
                                cudaMemcpyHostToDevice, sin), "cudaMemcpyAsync K") &&
           cuda(cudaMemcpyAsync(q + 2 * bytes + off, static_cast<const char*>(V_host) + off, len,
                                cudaMemcpyHostToDevice, sin), "cudaMemcpyAsync V") &&
           cuda(cudaEventRecord(e_in, sin), "cudaEventRecord") && cuda(cudaStreamWaitEvent(st, e_in, 0),
                                                                      "cudaStreamWaitEvent");
      if (!ok) break;
      pc.H = h1 - h0;
      pc.head_offset = hm.global(h0);
      g_launches = 0;
      const sparsepr_status s = forward_impl(&pc, q + off, q + bytes + off, q + 2 * bytes + off, o + off, nullptr,
                                             workspace, ws_bytes, stream, false);
      launches += g_launches;
      if (s != SPARSEPR_OK) { status = s; ok = false; break; }
      ok = cuda(cudaEventRecord(e_done, st), "cudaEventRecord") && cuda(cudaStreamWaitEvent(sout, e_done, 0),
                                                                        "cudaStreamWaitEvent") &&
           cuda(cudaMemcpyAsync(static_cast<char*>(O_host) + off, o + off, len, cudaMemcpyDeviceToHost, sout),
                "cudaMemcpyAsync O");
    }
    // `stream` completes only after the last copy out
    if (ok) ok = cuda(cudaEventRecord(e_end, sout), "cudaEventRecord") &&
                 cuda(cudaStreamWaitEvent(st, e_end, 0), "cudaStreamWaitEvent");
    g_launches = launches;
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  return status;
}

sparsepr_status sparsepr_dense_attention(const sparsepr_params* p, const void* Q, const void* K, const void* V,
                                         void* O, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  g_launches = 0;
  SPR_CHECK(check_params(p));
  SPR_TILED(Q); SPR_TILED(K); SPR_TILED(V); SPR_TILED(O);
  int* err = nullptr;
  const size_t need = p->frame_id ? 512 : 256;   // error word, then the frame ends
  if (workspace || p->frame_id) {
    if (!workspace || ((uintptr_t)workspace & 255) != 0 || ws_bytes < need)
      return failv(SPARSEPR_EWORKSPACE, "workspace must be 256-byte aligned and hold (bytes)", (long long)need);
    err = static_cast<int*>(workspace);
  }
  AttnArgs a{};
  a.Q = Q; a.K = K; a.V = V;
  a.BH = p->B * p->H; a.N = p->N; a.D = p->d;
  a.scale_log2 = eff_scale(*p) * 1.4426950408889634f;
  a.O = O; a.lse = lse; a.err = err;
  if (p->frame_id) {
    int* fend = at<int>(workspace, 256);
    SPR_LAUNCH(launch_frame_ends(p->frame_id, p->N, p->n_frames, fend, err, (cudaStream_t)stream));
    a.cz.frame_id = p->frame_id;
    a.cz.F = p->n_frames;
    a.cz.fend = fend;
  }
  SPR_LAUNCH(launch_attention_tc(a, true, (cudaStream_t)stream));
  return SPARSEPR_OK;
}

int sparsepr_workspace_error(const sparsepr_params* p, void* workspace, void* stream) {
  if (check_params(p) != SPARSEPR_OK || !workspace) return -1;
  int h = 0;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(&h, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return -1;
  if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
  return h;
}

sparsepr_status sparsepr_workspace_clear_error(const sparsepr_params* p, void* workspace, void* stream) {
  SPR_CHECK(check_params(p));
  SPR_NONNULL(workspace);
  cudaStream_t st = (cudaStream_t)stream;
  SPR_CUDA(cudaMemsetAsync(workspace, 0, 4, st));
  SPR_CUDA(cudaStreamSynchronize(st));
  return SPARSEPR_OK;
}

const char* sparsepr_status_string(sparsepr_status s) {
  switch (s) {
    case SPARSEPR_OK: return "ok";
    case SPARSEPR_EINVAL: return "invalid argument";
    case SPARSEPR_EUNSUPPORTED: return "unsupported configuration";
    case SPARSEPR_EWORKSPACE: return "workspace too small or misaligned";
    case SPARSEPR_ECUDA: return "CUDA error";
    case SPARSEPR_EDEVICE: return "device-side check failed";
  }
  return "unknown status";
}

const char* sparsepr_last_error(void) { return g_detail; }

int sparsepr_last_launch_count(void) { return g_launches; }

}  // extern "C"
