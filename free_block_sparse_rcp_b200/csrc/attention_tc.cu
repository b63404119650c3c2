// Route-walking flash attention on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Computes, for one q-tile of up to 128 permuted query rows of one query group,
//   O(q) = sum_{k routed} softmax(s q.k) v_k,   LSE(q) = ln sum_{k routed} exp(s q.k)
// (gist.science technical summary, section 2.C: attention over the routed cells of the
// group-contiguous layout), and writes O and LSE back to the original token positions.
//
// Roles of the 288 threads of a CTA:
//   warps 0-3  softmax + epilogue: thread t owns query row t = TMEM lane t
//   warp  4    TMEM allocation; lane 0 issues every tcgen05.mma
//   warps 5-8  gather: cp.async of the q rows and of the routed key/value rows of each
//              128-row chunk, by index through perm_q / perm_k, into 128B-swizzled
//              shared-memory tiles (the permuted layout is never materialised)
// Per chunk j:  S_j = Q K_j^T  -> TMEM (two buffers, so S_{j+1} overlaps softmax_j)
//               P_j = exp2(S_j * s*log2e - m) in bf16 -> shared memory (two buffers, so
//                     softmax_{j+1} overlaps PV_j)
//               O  += P_j V_j   (TMEM accumulator, rescaled in place only when a row's
//                                 running max grows by more than 2^8)
// Every mbarrier wait is bounded (2 s); a timeout raises an abort flag that ends every
// role, records DERR_WAIT_TIMEOUT in the workspace and still frees the TMEM.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace spr {
namespace tc {

constexpr int BM = 128;       // q rows per tile
constexpr int BN = 128;       // key rows per chunk
constexpr int NSOFT = 128;    // softmax threads (warps 0-3)
constexpr int MMA_WARP = 4;
constexpr int PROD0 = 160;    // first producer thread (warp 5)
constexpr int NPROD = 128;
constexpr int NT = 288;
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t q, full[2], empty[2], s_full[2], s_free[2], p_full[2], p_empty[2], o_done, mma_done;
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = (uint32_t)D * 128 * 2;  // Q / K / V tile bytes
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kTile;
  static constexpr uint32_t oV = oK + 2 * kTile;
  static constexpr uint32_t kP = 128 * 128 * 2;
  static constexpr uint32_t oP = oV + 2 * kTile;          // two P buffers
  static constexpr uint32_t oBar = oP + 2 * kP;
  static constexpr uint32_t oInt = oBar + 128;
};

template <int D, bool DENSE>
__global__ void __launch_bounds__(NT, 1)
    k_attn_tc(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
              const __nv_bfloat16* __restrict__ V, int N, int Gq, int Gk, const int* __restrict__ perm_q,
              const int* __restrict__ perm_k, const int* __restrict__ qoff, const int* __restrict__ koff,
              const int* __restrict__ rlist, const int* __restrict__ rcum, const int* __restrict__ rcnt,
              const int2* __restrict__ tiles, const int* __restrict__ tile_count, int max_tiles, float scale_log2,
              __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* err) {
  using L = Layout<D>;
  // The 128B-swizzled tiles need a 1024-byte aligned base; dynamic shared memory starts
  // at the CTA's shared window, which is aligned, and the layout leaves no room for a
  // realignment pad, so a misaligned base is reported and the tile skipped.
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
  int* sQrow = ints;                  // [128]
  int* sMisc = sQrow + 128;           // [0] tmem base, [1] abort, [2] total, [3] cnt, [4] slot ok
  int* sList = sMisc + 8;             // [Gk]
  int* sKoffL = sList + Gk;           // [Gk]
  int* sCum = sKoffL + Gk;            // [Gk + 1]
  volatile int* abort_flag = sMisc + 1;

  // ---------------- setup (all threads) ----------------
  int q0, qn;
  if (DENSE) {
    q0 = blockIdx.x * BM;
    if (q0 >= N) return;
    qn = min(BM, N - q0);
  } else {
    if ((int)blockIdx.x >= tile_count[bh]) return;
    const int2 tl = tiles[(size_t)bh * max_tiles + blockIdx.x];
    const int a = tl.x;
    const int* qo = qoff + (size_t)bh * (Gq + 1);
    q0 = qo[a] + tl.y * BM;
    qn = min(BM, qo[a + 1] - q0);
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
  if (DENSE && tid == 0) { sMisc[2] = N; sMisc[3] = 0; }
  if (tid < BM) {
    int row = -1;
    if (tid < qn) {
      row = DENSE ? q0 + tid : perm_q[head + q0 + tid];
      if (row < 0 || row >= N) { set_error(err, DERR_INDEX); row = -1; }
    }
    sQrow[tid] = row;
  }
  if (tid == 0) {
    sMisc[1] = 0;
    mbar_init(su32(&bars->q), NPROD);
    for (int s = 0; s < 2; ++s) {
      mbar_init(su32(&bars->full[s]), NPROD);
      mbar_init(su32(&bars->empty[s]), 1);
      mbar_init(su32(&bars->s_full[s]), 1);
      mbar_init(su32(&bars->s_free[s]), NSOFT);
      mbar_init(su32(&bars->p_full[s]), NSOFT);
      mbar_init(su32(&bars->p_empty[s]), 1);
    }
    mbar_init(su32(&bars->o_done), 1);
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
  const uint32_t sQ = base + L::oQ, sK = base + L::oK, sV = base + L::oV, sP = base + L::oP;
  const uint32_t tS0 = tmem, tO = tmem + 256;   // S buffers at columns 0 / 128, O at 256

  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  if (tid >= PROD0) {
    // ---------------- gather warps ----------------
    const int p = tid - PROD0;          // 0..127
    const int pl = p & 31, pw = p >> 5;
    constexpr int CPR = D / 8;          // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;       // rows per warp instruction
    // q rows
    for (int i = 0; i < 32 / RPI; ++i) {
      const int r = pw * 32 + i * RPI + pl / CPR, c = pl % CPR;
      const int row = sQrow[r];
      cp_async16(sQ + tile_off(r, c, 128), Q + (head + (row < 0 ? 0 : row)) * D + c * 8, row >= 0);
    }
    cp_async_arrive_noinc(su32(&bars->q));
    volatile int* prod_ok = sMisc + 4;
    for (int j = 0; j < nchunks; ++j) {
      const int s = j & 1;
      // one thread waits for the slot; the named barrier below publishes the outcome
      if (p == 0) *prod_ok = (j < 2 || wait(bars->empty[s], ((j >> 1) - 1) & 1)) ? 1 : 0;
      // key row of slot p of chunk j (this warp's 32 rows: 32 * pw + lane)
      int myrow = -1;
      {
        const int pos = j * BN + p;
        if (pos < total) {
          if (DENSE) {
            myrow = pos;
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
      named_sync(1, NPROD);
      if (!*prod_ok) break;
      const uint32_t dk = sK + s * L::kTile, dv = sV + s * L::kTile;
#pragma unroll
      for (int i = 0; i < 32 / RPI; ++i) {
        const int rl = i * RPI + pl / CPR, c = pl % CPR;   // row within this warp's 32
        const int row = __shfl_sync(0xffffffffu, myrow, rl);
        const int r = pw * 32 + rl;
        const size_t off = (head + (row < 0 ? 0 : row)) * D + c * 8;
        const uint32_t o = tile_off(r, c, 128);
        cp_async16(dk + o, K + off, row >= 0);
        cp_async16(dv + o, V + off, row >= 0);
      }
      cp_async_arrive_noinc(su32(&bars->full[s]));
    }
    cp_async_wait_all();
  } else if (warp == MMA_WARP) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(128, BN, false);
      constexpr uint32_t IDO = idesc_bf16(128, D, true);
      bool ok = nchunks == 0 || wait(bars->q, 0);
      auto issue_pv = [&](int i) -> bool {
        if (!wait(bars->p_full[i & 1], (i >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t vb = sV + (i & 1) * L::kTile;
        const uint32_t pb = sP + (i & 1) * L::kP;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t ad = sdesc(pb + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc(vb + k * 2048, 16384, 1024);
          tc_mma(tO, ad, bd, IDO, (i > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(su32(&bars->empty[i & 1]));
        tc_commit(su32(&bars->p_empty[i & 1]));
        tc_commit(su32(&bars->o_done));
        return true;
      };
      for (int j = 0; ok && j < nchunks; ++j) {
        const int s = j & 1;
        if (!wait(bars->full[s], (j >> 1) & 1)) { ok = false; break; }
        if (j >= 2 && !wait(bars->s_free[s], ((j >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK + s * L::kTile;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          tc_mma(tS0 + s * 128, sdesc(sQ + off, 16, 1024), sdesc(kb + off, 16, 1024), IDS, k > 0 ? 1u : 0u);
        }
        tc_commit(su32(&bars->s_full[s]));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nchunks > 0) issue_pv(nchunks - 1);
      // drain: every MMA issued above completes before the TMEM is released
      tc_commit(su32(&bars->mma_done));
      wait(bars->mma_done, 0);
    }
  } else {
    // ---------------- softmax + epilogue (thread t = row t) ----------------
    const int t = tid;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t sreg[128];
    for (int j = 0; j < nchunks; ++j) {
      const int b = j & 1;
      ok = wait(bars->s_full[b], (j >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      tc_ld128(tS0 + lane_off + b * 128, sreg);
      tc_fence_before();
      mbar_arrive(su32(&bars->s_free[b]));
      const int valid = total - j * BN;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c)
        if (c < valid) mx = fmaxf(mx, __uint_as_float(sreg[c]));
      const float m_new = fmaxf(m_used, mx * scale_log2);
      const bool need = (m_new > m_used + kRescaleThreshold) || (m_used == -INFINITY && m_new != -INFINITY);
      const bool warp_need = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (warp_need && m_new > m_used) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_new);
        m_used = m_new;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = c < valid ? ex2(__uint_as_float(sreg[c]) * scale_log2 - mu) : 0.f;
        const float p1 = c + 1 < valid ? ex2(__uint_as_float(sreg[c + 1]) * scale_log2 - mu) : 0.f;
        rs += p0 + p1;
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      l = l * alpha + rs;
      if (warp_need && j >= 1) {
        // O row *= alpha (in TMEM, warp-uniform) once PV_{j-1} has finished with it
        ok = __all_sync(0xffffffffu, wait(bars->o_done, (j - 1) & 1));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tc_ld32(tO + lane_off + c * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tc_st32(tO + lane_off + c * 32, o);
        }
      }
      if (j >= 2) {
        // P buffer b was last read by PV_{j-2}
        ok = __all_sync(0xffffffffu, wait(bars->p_empty[b], ((j >> 1) - 1) & 1));
        if (!ok) break;
      }
      // P row t -> shared memory ([2 halves][128 rows][64] bf16, 128B-swizzled)
      unsigned char* prow = smem + L::oP + b * L::kP;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + tile_off(t, c, 128)) = v;
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(su32(&bars->p_full[b]));
    }
    // epilogue
    const int row = sQrow[t];
    if (ok && nchunks > 0) {
      ok = wait(bars->o_done, (nchunks - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = O + (head + (row < 0 ? 0 : row)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        if (nchunks > 0) {
          tc_ld32(tO + lane_off + c * 32, o);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) tc_dealloc(tmem, TMEM_COLS);
}

}  // namespace tc

size_t attn_tc_smem_bytes(int D, int Gk) {
  const size_t tiles = (D == 64) ? tc::Layout<64>::oInt : tc::Layout<128>::oInt;
  size_t s = tiles + (size_t)(128 + 8 + 3 * Gk + 1) * 4;
  // at most one CTA per SM: the kernel allocates all 512 TMEM columns
  return s < 120 * 1024 ? 120 * 1024 : s;
}

template <int D, bool DENSE>
static cudaError_t launch_tc_t(const AttnArgs& a, cudaStream_t st) {
  const size_t sm = attn_tc_smem_bytes(D, DENSE ? 0 : a.Gk);
  auto kern = tc::k_attn_tc<D, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid(DENSE ? ceil_div(a.N, tc::BM) : a.max_tiles, a.BH);
  kern<<<grid, tc::NT, sm, st>>>((const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K, (const __nv_bfloat16*)a.V,
                                 a.N, a.Gq, a.Gk, a.perm_q, a.perm_k, a.qoff, a.koff, a.rlist, a.rcum, a.rcnt,
                                 a.tiles, a.tile_count, a.max_tiles, a.scale_log2, (__nv_bfloat16*)a.O, a.lse,
                                 a.err);
  return cudaGetLastError();
}

cudaError_t launch_attention_tc(const AttnArgs& a, bool dense, cudaStream_t st) {
  if (a.D == 64) return dense ? launch_tc_t<64, true>(a, st) : launch_tc_t<64, false>(a, st);
  return dense ? launch_tc_t<128, true>(a, st) : launch_tc_t<128, false>(a, st);
}

}  // namespace spr
