// Route-walking flash attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Computes, for the permuted query rows of one query group,
//   O(q) = sum_{k routed} softmax(s q.k) v_k,   LSE(q) = ln sum_{k routed} exp(s q.k)
// (gist.science technical summary, section 2.C: attention over the routed cells of the
// group-contiguous layout), and writes O and LSE back to the original token positions.
//
// One CTA takes a unit of up to 256 permuted query rows of one query group: two q-tiles
// of 128 rows that share one stream of routed key/value chunks, so every K/V chunk that
// reaches shared memory feeds two tiles and the tensor pipe always has one tile's MMAs to
// run while the other tile's softmax works.
//
// Roles of the threads:
//   warps 0-3   softmax + epilogue of tile 0: thread r owns query row r = TMEM lane r
//   warps 4-7   softmax + epilogue of tile 1
//   routed:  warps 8-11 gather by cp.async the q rows and the routed key/value rows of each
//            128-row chunk, by index through perm_q / perm_k, into 128B-swizzled shared-
//            memory tiles (the permuted layout is never materialised); warp 12 allocates
//            TMEM and its lane 0 issues every tcgen05.mma  (416 threads)
//   dense:   warp 8 loads 128-row boxes by TMA; warp 9 issues the MMAs  (320 threads)
// (TMA's four-row gather was measured far slower than the cp.async gather for the routed
// rows, so only the dense variant uses TMA.)
// TMEM (512 columns): tile t holds S_t at columns 256t .. 256t+127 and O_t at 256t+128 ..
// The softmax writes P_t = exp2(S_t * s log2e - m) as packed bf16 pairs over the first 64
// columns of S_t, and PV reads it straight from TMEM (A operand in tensor memory).
// Per chunk j the MMA issue order is  PV_0,j  S_0,j+1  PV_1,j  S_1,j+1: S_t,j+1 reuses the
// columns of P_t,j only after PV_t,j (tcgen05 MMAs of one thread execute in issue order),
// and when S_t,j+1 is complete so is PV_t,j, so the softmax may rescale O_t in place.
// The softmax makes one speculative pass per chunk against the running max (exponentials
// and their row sum, packed fp32x2 arithmetic) and keeps it while the chunk's row sum stays
// within 2^8 (so no probability exceeds 2^8); otherwise the chunk is redone against its
// own max and O is rescaled.
// Frame-causal variant (CAUSAL): a query of frame f sees only keys of frames <= f.  The
// key stream is then ordered so that the keys a frame-f row may use are a prefix of it:
// dense, the token order itself (frame ids are nondecreasing), prefix fend[f]; routed, the
// query group's causal stream (its routed K/V groups' keys frame by frame), prefix
// tlim[a][f].  A unit streams the prefix of its last row's frame; every row masks the
// columns past its own prefix, which only the few chunks straddling a row's limit need.
// K is staged in a 3-deep ring, V in a 2-deep ring.  Every mbarrier wait is bounded (2 s);
// a timeout raises an abort flag that ends every role, records DERR_WAIT_TIMEOUT in the
// workspace and still frees the TMEM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace spr {
namespace tc {

constexpr int BM = 128;       // q rows per tile
constexpr int TPC = 2;        // tiles per CTA
constexpr int BN = 128;       // key rows per chunk
constexpr int KST = 3;        // K ring depth
constexpr int VST = 2;        // V ring depth
constexpr int NSOFT = 128;    // softmax threads per tile
// dense: one TMA warp (8) + MMA warp (9); routed: four cp.async gather warps (8-11) + MMA
// warp (12)
constexpr int PROD_WARP = 8;
constexpr int NPROD_G = 128;   // gather threads of the routed variant
template <bool DENSE>
struct Roles {
  static constexpr int MMA_WARP = DENSE ? 9 : 12;
  static constexpr int NT = DENSE ? 320 : 416;
  static constexpr uint32_t kLoadArrivals = DENSE ? 1 : NPROD_G;   // arrivals per q / K / V stage
};
constexpr uint32_t TMEM_COLS = 512;
constexpr float kSpecSumBound = 256.0f;    // 2^8: largest row sum a speculative chunk may reach

struct Bars {
  uint64_t q, kfull[KST], kempty[KST], vfull[VST], vempty[VST], s_full[TPC], p_full[TPC], o_done[TPC], mma_done;
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = (uint32_t)D * 128 * 2;  // Q / K / V tile bytes
  static constexpr uint32_t oQ = 0;                          // TPC q tiles
  static constexpr uint32_t oK = oQ + TPC * kTile;
  static constexpr uint32_t oV = oK + KST * kTile;
  static constexpr uint32_t oBar = oV + VST * kTile;
  static constexpr uint32_t oInt = oBar + 256;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

template <int D, bool DENSE, bool CAUSAL>
__global__ void __launch_bounds__(Roles<DENSE>::NT, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
              const __grid_constant__ CUtensorMap tmv, const __nv_bfloat16* __restrict__ Q,
              const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V, int N, int Gq, int Gk,
              const int* __restrict__ perm_q,
              const int* __restrict__ perm_k, const int* __restrict__ qoff, const int* __restrict__ koff,
              const int* __restrict__ rlist, const int* __restrict__ rcum, const int* __restrict__ rcnt,
              const int2* __restrict__ tiles, const int* __restrict__ tile_count, int max_tiles, float scale_log2,
              const int* __restrict__ frame_id, const int* __restrict__ fend, const int* __restrict__ klist,
              const int* __restrict__ tlim, int F, __nv_bfloat16* __restrict__ O, float* __restrict__ lse,
              int* err) {
  using L = Layout<D>;
  constexpr int NT = Roles<DENSE>::NT;
  constexpr int MMA_WARP = Roles<DENSE>::MMA_WARP;
  // The 128B-swizzled tiles need a 1024-byte aligned base; dynamic shared memory starts
  // at the CTA's shared window, which is aligned, and the layout leaves no room for a
  // realignment pad, so a misaligned base is reported and the unit skipped.
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = su32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) set_error(err, DERR_INDEX);
    return;
  }

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const size_t head = (size_t)bh * N;

  Bars* bars = reinterpret_cast<Bars*>(smem + L::oBar);
  int* ints = reinterpret_cast<int*>(smem + L::oInt);
  int* sQrow = ints;                  // [TPC * BM]
  // [0] tmem base, [1] abort, [2] total, [3] cnt, [4] slot ok, [5] chunks of tile 0 (causal)
  int* sMisc = sQrow + TPC * BM;
  int* sList = sMisc + 8;             // [Gk]
  int* sKoffL = sList + Gk;           // [Gk]
  int* sCum = sKoffL + Gk;            // [Gk + 1]
  volatile int* abort_flag = sMisc + 1;

  // ---------------- setup (all threads) ----------------
  int q0, qn, a = 0;
  if (DENSE) {
    q0 = blockIdx.x * (TPC * BM);
    if (q0 >= N) return;
    qn = min(TPC * BM, N - q0);
  } else {
    if ((int)blockIdx.x >= tile_count[bh]) return;
    const int2 tl = tiles[(size_t)bh * max_tiles + blockIdx.x];
    a = tl.x;
    const int* qo = qoff + (size_t)bh * (Gq + 1);
    q0 = qo[a] + tl.y * (TPC * BM);
    qn = min(TPC * BM, qo[a + 1] - q0);
    if (!CAUSAL) {
      const int cnt = rcnt[(size_t)bh * Gq + a];
      const int* rl = rlist + ((size_t)bh * Gq + a) * Gk;
      const int* rc = rcum + ((size_t)bh * Gq + a) * (Gk + 1);
      const int* ko = koff + (size_t)bh * (Gk + 1);
      for (int i = tid; i < cnt; i += NT) {
        sList[i] = rl[i];
        sKoffL[i] = ko[rl[i]];
      }
      for (int i = tid; i <= cnt; i += NT) sCum[i] = rc[i];
      if (tid == 0) { sMisc[2] = rc[cnt]; sMisc[3] = cnt; }
    }
  }
  // per-frame key prefix of the stream: fend (dense) or this query group's tlim (routed)
  const int* frame_lim = CAUSAL ? (DENSE ? fend : tlim + ((size_t)bh * Gq + a) * F) : nullptr;
  auto frame_of = [&](int row) -> int {
    int f = (row >= 0 && row < N) ? frame_id[row] : F - 1;
    return f < 0 ? 0 : (f >= F ? F - 1 : f);
  };
  if (CAUSAL && tid == 0) {
    // the unit streams the prefix of its last (latest-frame) row; tile 0 stops at the
    // prefix of its own last row
    auto prefix_of = [&](int i) -> int {   // stream prefix of the frame of unit row i
      const int t = frame_lim[frame_of(DENSE ? q0 + i : perm_q[head + q0 + i])];
      return t < 0 ? 0 : (t > N ? N : t);
    };
    const int tot = qn > 0 ? prefix_of(qn - 1) : 0;
    sMisc[2] = tot;
    sMisc[3] = 0;
    sMisc[5] = qn > BM ? min((prefix_of(BM - 1) + BN - 1) / BN, (tot + BN - 1) / BN) : (tot + BN - 1) / BN;
  }
  if (DENSE && !CAUSAL && tid == 0) { sMisc[2] = N; sMisc[3] = 0; }
  if (tid < TPC * BM) {
    int row = -1;
    if (tid < qn) {
      row = DENSE ? q0 + tid : perm_q[head + q0 + tid];
      if (row < 0 || row >= N) { set_error(err, DERR_INDEX); row = -1; }
    }
    sQrow[tid] = row;
  }
  const int ntile = qn > BM ? 2 : 1;
  if (tid == 0) {
    sMisc[1] = 0;
    mbar_init(su32(&bars->q), Roles<DENSE>::kLoadArrivals);
    for (int s = 0; s < KST; ++s) {
      mbar_init(su32(&bars->kfull[s]), Roles<DENSE>::kLoadArrivals);
      mbar_init(su32(&bars->kempty[s]), 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(su32(&bars->vfull[s]), Roles<DENSE>::kLoadArrivals);
      mbar_init(su32(&bars->vempty[s]), 1);
    }
    for (int t = 0; t < TPC; ++t) {
      mbar_init(su32(&bars->s_full[t]), 1);
      mbar_init(su32(&bars->p_full[t]), NSOFT);
      mbar_init(su32(&bars->o_done[t]), 1);
    }
    mbar_init(su32(&bars->mma_done), 1);
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tc_alloc(su32(&sMisc[0]), TMEM_COLS);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];
  const int total = sMisc[2];
  const int cnt = sMisc[3];
  const int nchunks = (total + BN - 1) / BN;
  // chunks tile t walks: all (the last tile always walks every chunk), or fewer for tile 0
  // of a frame-causal unit, whose rows end in an earlier frame
  const int nch0 = CAUSAL ? sMisc[5] : nchunks;
  auto nch = [&](int t) -> int { return (CAUSAL && t == 0) ? nch0 : nchunks; };
  const uint32_t sQ = base + L::oQ, sK = base + L::oK, sV = base + L::oV;

  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  if (DENSE && warp == PROD_WARP) {
    // ---------------- TMA loads (one warp) ----------------
    bool ok = true;
    // q rows of both tiles (rows of an absent tile or past the group read row 0: never stored)
    if (lane == 0) mbar_arrive_expect_tx(su32(&bars->q), TPC * L::kTile);
    __syncwarp();
    if (lane < TPC * (D / 64)) {
      const int t = lane / (D / 64), h = lane % (D / 64);
      tma_load_2d(sQ + t * L::kTile + h * 16384, &tmq, 64 * h, (int)(head + q0 + BM * t), su32(&bars->q));
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      const int ks = j % KST, vs = j % VST;
      // K_j, V_j: rows j BN .. j BN + 127 of the head (rows past N are masked in the softmax)
      if (lane == 0) {
        ok = j < KST || wait(bars->kempty[ks], ((j / KST) - 1) & 1);
        if (ok) mbar_arrive_expect_tx(su32(&bars->kfull[ks]), L::kTile);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (lane < D / 64)
        tma_load_2d(sK + ks * L::kTile + lane * 16384, &tmk, 64 * lane, (int)(head + j * BN), su32(&bars->kfull[ks]));
      if (lane == 0) {
        ok = j < VST || wait(bars->vempty[vs], ((j / VST) - 1) & 1);
        if (ok) mbar_arrive_expect_tx(su32(&bars->vfull[vs]), L::kTile);
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if (lane < D / 64)
        tma_load_2d(sV + vs * L::kTile + lane * 16384, &tmv, 64 * lane, (int)(head + j * BN), su32(&bars->vfull[vs]));
    }
  } else if (!DENSE && warp >= PROD_WARP && warp < PROD_WARP + 4) {
    // ---------------- gather warps ----------------
    const int p = tid - PROD_WARP * 32;   // 0..127
    const int pl = p & 31, pw = p >> 5;
    constexpr int CPR = D / 8;          // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;       // rows per warp instruction
    // q rows of both tiles (rows of an absent tile are zero-filled)
    for (int i = 0; i < TPC * BM * CPR / NPROD_G; ++i) {
      const int e = i * NPROD_G + p;
      const int r = e / CPR, c = e % CPR;
      const int row = sQrow[r];
      cp_async16(sQ + (r / BM) * L::kTile + tile_off(r % BM, c, 128),
                 Q + (head + (row < 0 ? 0 : row)) * D + c * 8, row >= 0);
    }
    cp_async_arrive_noinc(su32(&bars->q));
    volatile int* prod_ok = sMisc + 4;
    for (int j = 0; j < nchunks; ++j) {
      // key row of slot p of chunk j (this warp's 32 rows: 32 * pw + lane)
      int myrow = -1;
      {
        const int pos = j * BN + p;
        if (pos < total) {
          if (DENSE) {
            myrow = pos;
          } else if (CAUSAL) {
            myrow = klist[((size_t)bh * Gq + a) * N + pos];
            if (myrow < 0 || myrow >= N) { set_error(err, DERR_INDEX); myrow = -1; }
          } else {
            int lo = 0, hi = cnt - 1;
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (sCum[mid] <= pos) lo = mid; else hi = mid - 1;
            }
            myrow = perm_k[head + sKoffL[lo] + (pos - sCum[lo])];
            if (myrow < 0 || myrow >= N) { set_error(err, DERR_INDEX); myrow = -1; }
          }
        }
      }
      // K_j -> ring slot j % KST (one thread waits; the named barrier publishes the outcome)
      const int ks = j % KST, vs = j % VST;
      if (p == 0) *prod_ok = (j < KST || wait(bars->kempty[ks], ((j / KST) - 1) & 1)) ? 1 : 0;
      named_sync(1, NPROD_G);
      if (!*prod_ok) break;
      {
        const uint32_t dk = sK + ks * L::kTile;
#pragma unroll
        for (int i = 0; i < 32 / RPI; ++i) {
          const int rl = i * RPI + pl / CPR, c = pl % CPR;   // row within this warp's 32
          const int row = __shfl_sync(0xffffffffu, myrow, rl);
          cp_async16(dk + tile_off(pw * 32 + rl, c, 128), K + (head + (row < 0 ? 0 : row)) * D + c * 8, row >= 0);
        }
      }
      cp_async_arrive_noinc(su32(&bars->kfull[ks]));
      // V_j -> ring slot j % VST
      named_sync(1, NPROD_G);   // every thread has read *prod_ok before it is rewritten
      if (p == 0) *prod_ok = (j < VST || wait(bars->vempty[vs], ((j / VST) - 1) & 1)) ? 1 : 0;
      named_sync(1, NPROD_G);
      if (!*prod_ok) break;
      {
        const uint32_t dv = sV + vs * L::kTile;
#pragma unroll
        for (int i = 0; i < 32 / RPI; ++i) {
          const int rl = i * RPI + pl / CPR, c = pl % CPR;
          const int row = __shfl_sync(0xffffffffu, myrow, rl);
          cp_async16(dv + tile_off(pw * 32 + rl, c, 128), V + (head + (row < 0 ? 0 : row)) * D + c * 8, row >= 0);
        }
      }
      cp_async_arrive_noinc(su32(&bars->vfull[vs]));
      named_sync(1, NPROD_G);   // *prod_ok is rewritten at the top of the next chunk
    }
    cp_async_wait_all();
  } else if (warp == MMA_WARP) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, BN, false);
      constexpr uint32_t IDO = idesc_bf16(128, D, true);
      bool ok = nchunks == 0 || wait(bars->q, 0);
      // the first tile that uses chunk j waits for its K / V stage
      auto first_user = [&](int j) -> int { return j < nch(0) ? 0 : 1; };
      // S_t,j = Q_t K_j^T into the S columns of tile t; the last tile releases K_j
      auto issue_s = [&](int t, int j) -> bool {
        const int ks = j % KST;
        if (t == first_user(j)) {
          if (!wait(bars->kfull[ks], (j / KST) & 1)) return false;
          tc_fence_after();
        }
        const uint32_t kb = sK + ks * L::kTile, qb = sQ + t * L::kTile;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          tc_mma(tmem + 256 * t, sdesc(qb + off, 16, 1024), sdesc(kb + off, 16, 1024), IDS, k > 0 ? 1u : 0u);
        }
        tc_commit(su32(&bars->s_full[t]));
        if (t == ntile - 1) tc_commit(su32(&bars->kempty[ks]));
        return true;
      };
      // O_t += P_t,j V_j with P_t,j read from TMEM; the last tile releases V_j
      auto issue_pv = [&](int t, int j) -> bool {
        const int vs = j % VST;
        if (!wait(bars->p_full[t], j & 1)) return false;
        if (t == first_user(j) && !wait(bars->vfull[vs], (j / VST) & 1)) return false;
        tc_fence_after();
        const uint32_t vb = sV + vs * L::kTile;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          tc_mma_ts(tmem + 256 * t + 128, tmem + 256 * t + k * 8, sdesc(vb + k * 2048, 16384, 1024), IDO,
                    (j > 0 || k > 0) ? 1u : 0u);
        if (t == ntile - 1) tc_commit(su32(&bars->vempty[vs]));
        return true;
      };
      for (int t = 0; ok && t < ntile; ++t)
        if (nch(t) > 0) ok = issue_s(t, 0);
      bool early0 = false;
      for (int j = 0; ok && j < nchunks; ++j) {
        for (int t = 0; ok && t < ntile; ++t) {
          if (j >= nch(t)) continue;
          ok = issue_pv(t, j);
          if (ok && j + 1 < nch(t)) ok = issue_s(t, j + 1);
          // a tile whose walk ends before the unit's releases its epilogue early
          if (ok && CAUSAL && t == 0 && ntile > 1 && j + 1 == nch(0)) {
            tc_commit(su32(&bars->o_done[0]));
            early0 = true;
          }
        }
      }
      for (int t = 0; t < ntile; ++t)
        if (!(t == 0 && early0)) tc_commit(su32(&bars->o_done[t]));
      // drain: every MMA issued above completes before the TMEM is released
      tc_commit(su32(&bars->mma_done));
      wait(bars->mma_done, 0);
    }
  } else if (warp < 4 * TPC) {
    // ---------------- softmax + epilogue (tile t, thread r = row r) ----------------
    const int t = warp >> 2;
    const int r = tid & (BM - 1);
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + 256 * t + lane_off, tO = tS + 128;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    // keys this row may use: the stream prefix of its frame (frame-causal), else all
    int lim = total;
    if (CAUSAL) {
      const int row = sQrow[t * BM + r];
      if (row >= 0) lim = min(total, frame_lim[frame_of(row)]);
    }
    const int nct = t < ntile ? nch(t) : 0;   // chunks this tile walks
    if (t < ntile) {
      uint32_t sreg[64];
      uint32_t pk[64];
      const uint64_t sc2 = f2pack(scale_log2, scale_log2);
      for (int j = 0; j < nct; ++j) {
        ok = __all_sync(0xffffffffu, wait(bars->s_full[t], j & 1));
        if (!ok) break;
        tc_fence_after();
        const int valid = lim - j * BN;
        const bool full = CAUSAL ? __all_sync(0xffffffffu, valid >= BN) : valid >= BN;
        // Speculative single pass against the running max: P = exp2(S s log2e - m) and its
        // row sum; kept only if that sum stays within kSpecSumBound.
        bool need = true;
        float mx = -INFINITY;
        uint64_t rs2 = 0ull;
        const bool spec = __all_sync(0xffffffffu, m_used != -INFINITY);
        if (spec) {
          const uint64_t nmu2 = f2pack(-m_used, -m_used);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tc_ld32(tS + 32 * q, sreg);
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float s0 = __uint_as_float(sreg[c]), s1 = __uint_as_float(sreg[c + 1]);
              if (!full) {
                if (32 * q + c >= valid) s0 = -INFINITY;
                if (32 * q + c + 1 >= valid) s1 = -INFINITY;
              }
              float x0, x1;
              f2unpack(ffma2(f2pack(s0, s1), sc2, nmu2), x0, x1);
              const float p0 = ex2(x0), p1 = ex2(x1);
              rs2 = fadd2(rs2, f2pack(p0, p1));
              pk[16 * q + (c >> 1)] = pack_bf16(p0, p1);
            }
          }
          // kept iff the chunk's row sum stays <= 2^8, which bounds every element by 2^8
          // (no per-element max is kept)
          float r0, r1;
          f2unpack(rs2, r0, r1);
          need = !(r0 + r1 <= kSpecSumBound);
        }
        const bool warp_need = __any_sync(0xffffffffu, need);
        float alpha = 1.f;
        if (!warp_need) {
          // keys 64h .. 64h+63 -> packed P in columns 32h .. 32h+31 (all S of the chunk read)
          tc_st32(tS, pk);
          tc_st32(tS + 32, pk + 32);
          float r0, r1;
          f2unpack(rs2, r0, r1);
          l += r0 + r1;
        } else {
          // slow path: the chunk's max, rescale O, then P against it
          {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              tc_ld64(tS + 64 * h, sreg);
              float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
              for (int c = 0; c < 64; ++c)
                if (64 * h + c < valid) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(sreg[c]));
              mx = fmaxf(mx, fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])));
            }
          }
          const float m_new = fmaxf(m_used, mx * scale_log2);
          if (m_new > m_used) {
            alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_new);
            m_used = m_new;
          }
          if (j >= 1) {
            // O row *= alpha in TMEM: PV_t,j-1 completed before S_t,j did
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tc_ld32(tO + c * 32, o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tc_st32(tO + c * 32, o);
            }
          }
          const float mu = (m_used == -INFINITY) ? 0.f : m_used;
          float rs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tc_ld64(tS + 64 * h, sreg);
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float p0 = 64 * h + c < valid ? ex2(__uint_as_float(sreg[c]) * scale_log2 - mu) : 0.f;
              const float p1 = 64 * h + c + 1 < valid ? ex2(__uint_as_float(sreg[c + 1]) * scale_log2 - mu) : 0.f;
              rs[(c >> 1) & 3] += p0 + p1;
              pk[c >> 1] = pack_bf16(p0, p1);
            }
            tc_st32(tS + 32 * h, pk);
          }
          l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
        }
        tc_fence_before();
        mbar_arrive(su32(&bars->p_full[t]));
      }
      // epilogue
      const int row = sQrow[t * BM + r];
      if (ok && nct > 0) ok = __all_sync(0xffffffffu, wait(bars->o_done[t], 0));
      if (ok) {
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* orow = O + (head + (row < 0 ? 0 : row)) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (nct > 0) {
            tc_ld32(tO + c * 32, o);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
          if (row >= 0) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
        if (row >= 0 && lse) lse[head + row] = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) tc_dealloc(tmem, TMEM_COLS);
}

}  // namespace tc

size_t attn_tc_smem_bytes(int D, int Gk) {
  const size_t tiles = (D == 64) ? tc::Layout<64>::oInt : tc::Layout<128>::oInt;
  size_t s = tiles + (size_t)(tc::TPC * tc::BM + 8 + 3 * Gk + 1) * 4;
  // at most one CTA per SM: the kernel allocates all 512 TMEM columns
  return s < 120 * 1024 ? 120 * 1024 : s;
}

template <int D, bool DENSE, bool CAUSAL>
static cudaError_t launch_tc_t(const AttnArgs& a, cudaStream_t st) {
  const size_t sm = attn_tc_smem_bytes(D, DENSE ? 0 : a.Gk);
  auto kern = tc::k_attn_tc<D, DENSE, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  // tensor maps of 128-row boxes (used by the dense variant only)
  CUtensorMap tq{}, tk{}, tv{};
  if (DENSE) {
    const unsigned long long rows = (unsigned long long)a.BH * a.N;
    if ((e = make_tmap_bf16_rows(&tq, a.Q, rows, D, tc::BM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&tk, a.K, rows, D, tc::BM)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16_rows(&tv, a.V, rows, D, tc::BM)) != cudaSuccess) return e;
  }
  dim3 grid(DENSE ? ceil_div(a.N, tc::TPC * tc::BM) : a.max_tiles, a.BH);
  kern<<<grid, tc::Roles<DENSE>::NT, sm, st>>>(tq, tk, tv, (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K,
                                               (const __nv_bfloat16*)a.V, a.N, a.Gq, a.Gk, a.perm_q, a.perm_k, a.qoff,
                                               a.koff, a.rlist, a.rcum, a.rcnt, a.tiles, a.tile_count, a.max_tiles,
                                               a.scale_log2, a.cz.frame_id, a.cz.fend, a.cz.klist, a.cz.tlim, a.cz.F,
                                               (__nv_bfloat16*)a.O, a.lse, a.err);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_tc_d(const AttnArgs& a, bool dense, cudaStream_t st) {
  if (a.cz.on()) return dense ? launch_tc_t<D, true, true>(a, st) : launch_tc_t<D, false, true>(a, st);
  return dense ? launch_tc_t<D, true, false>(a, st) : launch_tc_t<D, false, false>(a, st);
}

cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, cudaStream_t st) {
  return a.D == 64 ? launch_tc_d<64>(a, dense, st) : launch_tc_d<128>(a, dense, st);
}

}  // namespace spr
