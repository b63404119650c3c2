/*
 * sparsepr.h -- C ABI of the SparsePR per-call sparse-attention library (sm_100a).
 *
 * SparsePR ("Partition the Support, Reconstruct the Residual", arXiv 2608.18484)
 * replaces one softmax attention call O = softmax(s Q K^T) V by
 *   1. a response-coupled partition of keys and queries into groups
 *      (gist.science technical summary, section 2.A),
 *   2. a budgeted route of (query group, K/V group) cells and a group-contiguous
 *      permutation (same page, section 2.C; huashangw.com article, section on
 *      sparse execution),
 *   3. attention restricted to the routed cells (section 2.C),
 *   4. exact attention for 64 query-group-stratified probe rows per head, a ridge
 *      affine fit R ~ b + xB of the probe residuals inside their top singular
 *      subspace (section 2.B; huashangw.com method walkthrough), and
 *   5. the correction of every unprobed row (section 2.B).
 * The call takes Q, K, V and a target executed-pair density and returns the
 * reconstructed output (ai-feeds.com summary, 方法: 输入 / 输出).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are device pointers unless stated.  Q, K, V and outputs named O* are
 *    bf16, contiguous [B, H, N, d] (row stride d elements), and start on a 16-byte
 *    boundary (the kernels move them with TMA; a misaligned one is SPARSEPR_EINVAL).
 *    "BH" below is B*H and every per-head array is laid out head-major ([B, H, ...]
 *    flattened).
 *  - Token indices are int32 positions in [0, N) of the original sequence.
 *  - Ownership: the caller owns every buffer.  Every entry point except
 *    sparsepr_probe_fit_noalloc allocates nothing and keeps no state between calls:
 *    their scratch memory is the caller's `workspace` (device, 256-byte aligned, at
 *    least sparsepr_workspace_bytes(p) bytes); partition, attend and probe_fit use
 *    disjoint regions of it, so attend and probe_fit may run concurrently on two
 *    streams sharing one workspace.  sparsepr_probe_fit_noalloc instead uses a fixed
 *    16 MiB device array that the library holds on every GPU that loads it (see its
 *    declaration).  sparsepr_forward (and the host entry points built on it) creates
 *    and releases a second stream and CUDA events inside the call, and
 *    sparsepr_forward_host_chunked its CUDA events (no device memory).
 *  - Asynchrony: every call only enqueues work on `stream` (a cudaStream_t; NULL
 *    is the legacy default stream) and returns.  Argument errors are detected on
 *    the host before anything is enqueued and return SPARSEPR_EINVAL or
 *    SPARSEPR_EUNSUPPORTED; a failed launch returns SPARSEPR_ECUDA.  Device-side
 *    checks (bounded waits, index checks) record an error code in the workspace;
 *    read it with sparsepr_workspace_error() after the stream has drained.  Codes:
 *    1 index out of range, 2 bounded wait ran out, 3 random-draw map overflow,
 *    4 non-finite value, 5 frame ids out of range or decreasing, 6 more than 2048
 *    k-means label corrections for one block of 16 groups in one Lloyd step (the
 *    exact re-check of near-tie rows; the call's outputs are then unspecified).
 *  - Determinism: for fixed inputs, params and seed every output is bitwise
 *    reproducible (no floating-point atomics on any output path).
 *  - Random draws (query sample, k-means seeds, probe rows) use SplitMix64
 *    (Steele, Lea & Flood 2014) with one stream per (head, purpose):
 *    state0 = mix(seed + 0xD1B54A32D192ED03 * (8*g + purpose + 1)),
 *    purpose 0 = query sample, 1 = key k-means seeds, 2 = query k-means seeds,
 *    3 = probe rows; a draw of m of n items is a partial Fisher-Yates shuffle
 *    (j = i + next() mod (n - i)).  g is the head's index in the whole layer:
 *    g = b * heads_total + head_offset + h for head h of batch element b of the
 *    call (g = b * H + h by default), so a call split by heads or batch elements
 *    (over GPUs, or in chunks) reproduces the unsplit call bit for bit.
 */
#ifndef SPARSEPR_H
#define SPARSEPR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPARSEPR_API __attribute__((visibility("default")))
#else
#define SPARSEPR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARSEPR_OK = 0,
  SPARSEPR_EINVAL = 1,        /* invalid argument (null pointer, size out of range, density below the probe floor) */
  SPARSEPR_EUNSUPPORTED = 2,  /* valid but outside what the kernels implement (d not 64/128, too many groups, ...) */
  SPARSEPR_EWORKSPACE = 3,    /* workspace smaller than sparsepr_workspace_bytes() or misaligned */
  SPARSEPR_ECUDA = 4,         /* a CUDA runtime call or kernel launch failed */
  SPARSEPR_EDEVICE = 5        /* a device-side check failed (see sparsepr_workspace_error) */
} sparsepr_status;

/* Parameters of one attention call.  Defaults that the pages leave open are
 * readings; the recommended values per workload are listed with each field. */
typedef struct {
  int B, H, N, d;          /* batch, heads, tokens, head dim (d = 64 or 128)                        */
  int block;               /* tile rows of the permuted layout reported in block_mask (64 or 128)  */
  float density;           /* target executed-pair density rho_exec in (0, 1], probe pairs included;
                              >= 1 routes every non-empty cell                                      */
  int n_kgroups;           /* K/V groups G_k: 1..min(N,1024) is valid (else SPARSEPR_EINVAL); the
                              kernels implement G_k <= 128, more returns SPARSEPR_EUNSUPPORTED     */
  int n_qgroups;           /* query groups G_q: as G_k (valid up to min(N,1024), implemented up to
                              128)                                                                 */
  int n_samples;           /* sampled queries M_s for M_K (1..min(N,1024); default max(64, d))      */
  int n_probes;            /* probe rows per head P (1..min(N,64); the article uses 64)             */
  int eig_rank;            /* eigenpairs of M_K kept for key coordinates r_e (16 or 32; default d/4) */
  int sub_rank;            /* probe-residual subspace rank r (1..min(d, P, 64))                     */
  int kmeans_iters;        /* Lloyd assignment steps per k-means (1..64)                            */
  float ridge_lambda;      /* ridge penalty, absolute (> 0; default 1e-2)                           */
  float scale;             /* softmax scale; 0 means 1/sqrt(d)                                      */
  unsigned long long seed; /* seed of the SplitMix64 streams                                        */
  const int* frame_id;     /* NULL, or device int32 [N]: frame of each token (shared by all b, h);
                              then query q sees key k only if frame_id[k] <= frame_id[q]
                              (frame-causal, intersected with the route; the cell mass, cell cost
                              and budget count visible pairs only).  Ids must be nondecreasing in
                              token order (frame-major flattening of a video latent) and lie in
                              [0, n_frames); a violation is recorded as device error 5 and leaves
                              the outputs unspecified.  Needs N <= 65535 (32-bit cell costs).     */
  int n_frames;            /* with frame_id: number of frames, 1..64; ignored without frame_id     */
  int partition_mode;      /* 0: response-coupled partition (the method);
                              1: the semantic-grouping baseline of the pages' comparison (keys and
                              queries clustered separately on their raw vectors, same k-means
                              rules, seed streams, centroids, route and layout).  In mode 1 the
                              trace's sample_idx, metric, eigval, eigvec and key_coords are not
                              written.                                                            */
  int fit_weighted;        /* 0: uniform probe weights in the ridge fit; 1: each probe weighted by
                              n_a / (probes of its group a), normalised to mean 1 (the weighted
                              affine fit one page mentions)                                       */
  int fit_input;           /* input x of the affine map R ~ b + xB:
                              0 (default): the row's whole d-dimensional sparse output, with only
                              the correction projected onto the residual subspace (gist.science
                              2.B; huashangw.com method section: the corrected result is limited
                              to the residual directions the probes observed);
                              1: the sparse output projected on that subspace as well (x V_r)    */
  int head_offset;         /* index of this call's first head in the layer (>= 0; default 0)      */
  int heads_total;         /* heads per batch element of the layer (0: H; else >= head_offset + H);
                              with head_offset only the random streams depend on them              */
} sparsepr_params;

/* Optional debug copies of partition intermediates (any pointer may be NULL). */
typedef struct {
  int* sample_idx;          /* [BH, M_s]            sampled query rows, draw order                  */
  float* metric;            /* [BH, d, d]           M_K = Q_s^T Q_s / M_s                           */
  float* eigval;            /* [BH, r_e]            leading eigenvalues, descending                 */
  float* eigvec;            /* [BH, d, r_e]         matching eigenvectors (columns)                 */
  float* key_coords;        /* [BH, N, r_e]         y = Lambda^{1/2} U^T k                          */
  int* key_init;            /* [BH, G_k]            k-means seed rows                               */
  int* key_label_iters;     /* [T, BH, N]           key labels after every assignment step          */
  float* key_centroids;     /* [BH, G_k, d]         mean raw key per K/V group                      */
  float* query_coords;      /* [BH, N, G_k]         z = s C q                                       */
  int* query_init;          /* [BH, G_q]                                                            */
  int* query_label_iters;   /* [T, BH, N]                                                           */
  float* cell_mass;         /* [BH, G_q, G_k]       estimated retained mass per cell                */
  double* alpha;            /* [BH]                 shared mass target chosen by the route          */
} sparsepr_partition_trace;

/* Optional debug copies of probe intermediates (any pointer may be NULL). */
typedef struct {
  float* probe_o_sparse;    /* [BH, P, d]  routed-only output of the probe rows (fp32)              */
  float* probe_lse_dense;   /* [BH, P]     natural-log partition functions                          */
  float* probe_lse_sparse;  /* [BH, P]                                                              */
  float* sigma;             /* [BH, r]     singular values of the probe residual matrix             */
  float* b_sub;             /* [BH, r]     intercept in subspace coordinates                        */
} sparsepr_probe_trace;

/* Bytes of device workspace any call below needs for these params (0 if the
 * params are invalid or unsupported). */
SPARSEPR_API size_t sparsepr_workspace_bytes(const sparsepr_params* p);

/* Host-only validation of the params (no CUDA call). */
SPARSEPR_API sparsepr_status sparsepr_validate(const sparsepr_params* p);

/* Response-coupled partition, route and permutation
 * (gist.science 2.A and 2.C; huashangw.com, method and sparse-execution sections).
 *   Q, K       bf16 [B, H, N, d]
 *   perm_q/k   int32 [BH, N]     permuted position -> original token (stable by group)
 *   label_q/k  int32 [BH, N]     group of each original token
 *   qoff/koff  int32 [BH, G+1]   first permuted position of each group
 *   route      uint8 [BH, G_q, G_k]  1 = cell executed
 *   block_mask uint8 [BH, T, T]  T = ceil(N/block); tile (i, j) of the permuted layout holds a routed pair
 *   rho_exec   float [BH]        realized (routed pairs + P*N) / N^2; frame-causal: (routed visible
 *                                pairs + P*V/N) / V with V the visible pairs of the causal mask
 *   trace      optional, may be NULL                                                   */
SPARSEPR_API sparsepr_status sparsepr_partition(const sparsepr_params* p, const void* Q, const void* K,
                                   int* perm_q, int* perm_k, int* label_q, int* label_k,
                                   int* qoff, int* koff, unsigned char* route,
                                   unsigned char* block_mask, float* rho_exec,
                                   const sparsepr_partition_trace* trace,
                                   void* workspace, size_t ws_bytes, void* stream);

/* Attention restricted to the routed cells (gist.science 2.C):
 *   O_sparse(q) = sum over keys k with route[label_q(q), label_k(k)] of softmax(s q.k) v_k,
 * written in ORIGINAL token order (bf16 [B, H, N, d]); lse = ln sum exp(s q.k) over the
 * same keys (float [BH, N]).  Inputs are the partition outputs above.                 */
SPARSEPR_API sparsepr_status sparsepr_attend(const sparsepr_params* p, const void* Q, const void* K,
                                const void* V, const int* perm_q, const int* perm_k,
                                const int* qoff, const int* koff, const unsigned char* route,
                                void* O_sparse, float* lse,
                                void* workspace, size_t ws_bytes, void* stream);

/* Exact probes and the residual fit (gist.science 2.B; huashangw.com method section).
 *   probe_idx      int32 [BH, P]    probe rows (original indices), group order then draw order
 *   probe_o_dense  float [BH, P, d] exact dense output of the probe rows
 *   b_full         float [BH, d]    b V_r^T (intercept in output space)
 *   Vr             float [BH, d, r] orthonormal basis of the residual subspace (zero columns
 *                                   where the singular value is <= 1e-6 of the largest)
 *   W              float [BH, d, r] ridge slope, residual coordinates = x W
 *   Bmat           float [BH, d, d] optional (may be NULL): the pages' B = W V_r^T
 * Depends only on the partition (not on sparsepr_attend's output).                     */
SPARSEPR_API sparsepr_status sparsepr_probe_fit(const sparsepr_params* p, const void* Q, const void* K,
                                   const void* V, const int* label_k, const int* perm_q,
                                   const int* qoff, const unsigned char* route,
                                   int* probe_idx, float* probe_o_dense, float* b_full,
                                   float* Vr, float* W, float* Bmat,
                                   const sparsepr_probe_trace* trace,
                                   void* workspace, size_t ws_bytes, void* stream);

/* sparsepr_probe_fit without a workspace: allocates nothing and uses no caller scratch.
 * The paper has no counterpart; this variant exists for callers that cannot call
 * cudaMalloc (runtimes that fix their device memory plan at start-up and forbid later
 * allocation, or host code where an allocation, which can synchronize the device, is not
 * allowed).  Arguments and outputs are those of sparsepr_probe_fit minus the trace and the
 * workspace; results agree with it up to floating-point summation order.
 * Frame-causal params (frame_id != NULL) are refused with SPARSEPR_EUNSUPPORTED, and Q, K,
 * V must be 16-byte aligned (else SPARSEPR_EINVAL), both before any work is enqueued.
 * Scratch: a 16 MiB device array owned by the library, present on every GPU that loads
 * it until the process exits.  With S key splits it holds
 *   B*H*(n_probes*(4*d + 12) + S*64*(8*d + 16)) bytes (each region rounded up to 256)
 * plus a 256-byte error word; S starts at the workspace entry point's split count for N
 * and shrinks until the problem fits, and a problem that does not fit even with S = 1
 * returns SPARSEPR_EUNSUPPORTED before any work is enqueued.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress, with that device current)
 * and keeps it for the life of the process (a cudaDeviceReset invalidates it); make that
 * first call before any stream capture.  All calls share the one array and it keeps the
 * previous call's contents: the call clears its error word and rewrites every other byte
 * before reading it; calls that overlap on the GPU, on other streams or from other host
 * threads, race and must be serialized by the caller.  A device-side failure (a bounded
 * wait that ran out, an index out of range, a failed random draw) sets b_full, Vr, W and
 * Bmat of every head to NaN instead of leaving stale values.                           */
SPARSEPR_API sparsepr_status sparsepr_probe_fit_noalloc(const sparsepr_params* p, const void* Q,
                                                        const void* K, const void* V,
                                                        const int* label_k, const int* perm_q,
                                                        const int* qoff, const unsigned char* route,
                                                        int* probe_idx, float* probe_o_dense,
                                                        float* b_full, float* Vr, float* W,
                                                        float* Bmat, void* stream);

/* Correction of every unprobed row and restoration of the probe rows (gist.science 2.B):
 *   O(q) = x + b_full + (x W) V_r^T   with x = O_sparse(q), for q not a probe;
 *   O(q) = probe_o_dense              for probe rows.
 * O is bf16 [B, H, N, d] and may alias O_sparse.                                       */
SPARSEPR_API sparsepr_status sparsepr_reconstruct(const sparsepr_params* p, const void* O_sparse,
                                     const int* probe_idx, const float* probe_o_dense,
                                     const float* b_full, const float* Vr, const float* W,
                                     void* O, void* stream);

/* The whole call (partition -> attend -> probe_fit -> reconstruct) on device buffers,
 * with every intermediate kept in the workspace (sparsepr_forward_workspace_bytes).
 * rho_exec (float [BH]) may be NULL.  The probe path (sparsepr_probe_fit's kernels) runs
 * on a second stream that the call creates, forks from `stream` after the partition and
 * joins back before the correction, so it overlaps the routed attention; the stream and
 * its events are released before the call returns (freed once their work completes).
 * If they cannot be created, or `stream` is being captured into a CUDA graph, everything
 * runs on `stream`.  The results do not depend on the overlap.                         */
SPARSEPR_API size_t sparsepr_forward_workspace_bytes(const sparsepr_params* p);
SPARSEPR_API sparsepr_status sparsepr_forward(const sparsepr_params* p, const void* Q, const void* K,
                                 const void* V, void* O, float* rho_exec,
                                 void* workspace, size_t ws_bytes, void* stream);

/* sparsepr_forward from HOST buffers: copies Q, K, V (host, bf16 [B,H,N,d]; pinned memory
 * for asynchronous copies) into the caller's device staging buffer qkv_dev (3 tensors,
 * 3*BH*N*d bf16), runs the call into o_dev (device, bf16), and copies the result to
 * O_host.  Everything is enqueued on `stream`; the caller synchronizes.               */
SPARSEPR_API sparsepr_status sparsepr_forward_host(const sparsepr_params* p, const void* Q_host,
                                      const void* K_host, const void* V_host, void* O_host,
                                      void* qkv_dev, void* o_dev,
                                      void* workspace, size_t ws_bytes, void* stream);

/* sparsepr_forward_host as a pipeline over head chunks, so that the host<->device copies
 * of one chunk run beside the compute of another.  The B*H heads (flattened b*H + h) are
 * split into n_chunks (1..min(B*H, 512)) consecutive ranges of ceil(B*H / n_chunks) heads
 * (with head_offset / heads_total set, also at every batch element).  Chunk c's three
 * host-to-device copies (one cudaMemcpyAsync per tensor) go on copy_in_stream, its call
 * (sparsepr_forward with B = 1 over the chunk's heads, head_offset = their layer index, so
 * every output equals the unsplit call's bit for bit) on `stream`, and the copy of its O
 * back to O_host on copy_out_stream.  The copies in start after the work already enqueued
 * on `stream`; `stream` completes after the last copy out, so synchronizing `stream` is
 * enough.  A NULL copy stream means `stream` (no overlap).
 *   qkv_dev   device bf16 [3][B, H, N, d] staging of Q, K, V; o_dev device bf16 [B, H, N, d]
 *   workspace sparsepr_forward_workspace_bytes of the params of one chunk (B = 1,
 *             H = ceil(B*H / n_chunks)), shared by the chunks (their compute is serialized
 *             on `stream`); its error word is cleared once and collects every chunk's
 *             device errors
 * Host buffers should be pinned for the copies to be asynchronous.  The call creates its
 * CUDA events and releases them before returning (they are freed once they complete).  */
SPARSEPR_API sparsepr_status sparsepr_forward_host_chunked(const sparsepr_params* p, const void* Q_host,
                                                           const void* K_host, const void* V_host,
                                                           void* O_host, void* qkv_dev, void* o_dev,
                                                           int n_chunks, void* workspace, size_t ws_bytes,
                                                           void* stream, void* copy_in_stream,
                                                           void* copy_out_stream);

/* Dense softmax attention on the same machinery (the comparator for the sparse call):
 * O = softmax(s Q K^T) V (bf16 [B,H,N,d]), lse float [BH, N] (may be NULL); with frame ids,
 * each query attends to the keys of its own and earlier frames.  Uses only the first bytes
 * of the workspace: the error word (256 bytes; the workspace may then be NULL) and, with
 * frame ids, the frame ends (512 bytes in all, required).                              */
SPARSEPR_API sparsepr_status sparsepr_dense_attention(const sparsepr_params* p, const void* Q,
                                         const void* K, const void* V, void* O, float* lse,
                                         void* workspace, size_t ws_bytes, void* stream);

/* Device-side error code recorded in the workspace (0 = none) and its reset.  The code
 * is sticky until cleared; sparsepr_partition and sparsepr_forward clear it when they
 * start.  Both functions synchronize `stream`.                                         */
SPARSEPR_API int sparsepr_workspace_error(const sparsepr_params* p, void* workspace, void* stream);
SPARSEPR_API sparsepr_status sparsepr_workspace_clear_error(const sparsepr_params* p, void* workspace,
                                               void* stream);

/* Human-readable status; sparsepr_last_error() gives the detail of the most recent
 * failing call on this host thread (static storage, never NULL).                      */
SPARSEPR_API const char* sparsepr_status_string(sparsepr_status s);
SPARSEPR_API const char* sparsepr_last_error(void);

/* Number of kernel launches the last successful call on this host thread enqueued. */
SPARSEPR_API int sparsepr_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* SPARSEPR_H */
