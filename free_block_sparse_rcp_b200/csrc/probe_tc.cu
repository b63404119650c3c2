// Exact probe rows on the tensor cores (gist.science technical summary, section 2.B:
// probe rows evaluated exactly, R = O_dense - O_sparse).
//
// One CTA = the (up to 64) probe rows of one head against one contiguous key split.  The
// 128-row MMA tile holds every probe row twice: rows 0-63 take the softmax over all keys
// (dense), rows 64-127 the softmax over the keys whose K/V group is routed for the probe
// row's query group (sparse).  So for every 128-key chunk one S = Q K^T gives both, one
// set of PV MMAs accumulates both O_dense (rows 0-63) and O_sparse (rows 64-127) in TMEM,
// and each of the four softmax warps (one per TMEM sub-partition) has real rows.  The
// probabilities are kept to ~2^-17 by splitting them into bf16 hi + lo, both written to
// TMEM and both used as the A operand of the PV MMAs, so the probe outputs carry
// fp32-level error, not bf16's.  Each split writes base-2 running maxima, sums and
// unnormalised outputs in fp32; the combine kernel merges the splits.
//
// Roles (576 threads): warps 0-15 softmax, warp = quarter * 4 + row group: thread = tile row
// (row group * 32 + lane = TMEM lane) x 32-key quarter of the chunk; the four quarters of a
// row exchange their maxima once per chunk (mbarrier) and keep separate partial sums,
// added at the end.  Warp 16: TMEM allocation + MMA issue (lane 0).  Warp 17: loads -- the
// probe rows (cp.async, gathered through probe_idx), the K chunks with their key labels and
// the V chunks (TMA, two-deep rings of their own: a K stage is refilled as soon as its S
// MMAs completed and every softmax warp built its key mask from the labels, a V stage once
// its PV MMAs completed, so the next chunk's keys arrive while this one is in the softmax).
// The softmax warps arrive on the barriers once per warp.  A sparse row's key mask is built
// from the labels read 16 bytes at a time against the routed-group bits of its query group.
// TMEM: S at columns 0 / 128 (two buffers), P hi at 256, P lo at 320, O at 384.
// All waits bounded.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace spr {
namespace ptc {

using namespace spr::tc;

constexpr int BM = 128;    // tile rows: probe rows (dense) then probe rows again (sparse)
constexpr int PROWS = 64;  // probe rows per split (matches the combine's layout)
constexpr int BN = 128;    // keys per chunk
constexpr int NSOFT = 512;   // softmax threads
constexpr int MMA_WARP = 16;
constexpr int LOAD_WARP = 17;
constexpr int NT = 576;
constexpr float kRescaleThreshold = 8.0f;

struct Bars {
  uint64_t q, full[2], empty[2], vfull[2], vempty[2], s_full[2], s_free[2], p_full, p_empty, o_done, mma_done, mready[2], ldone;
};

template <int D>
struct Layout {
  static constexpr uint32_t kQ = (uint32_t)BM * D * 2;    // Q tile
  static constexpr uint32_t kKV = (uint32_t)BN * D * 2;   // one K or V chunk
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kQ;
  static constexpr uint32_t oV = oK + 2 * kKV;
  static constexpr uint32_t oLab = oV + 2 * kKV;           // int [2][BN]
  static constexpr uint32_t oXm = oLab + 2 * BN * 4;       // float [2][4][BM] quarter maxima, [4][BM] sums
  static constexpr uint32_t oBar = oXm + 3 * 4 * BM * 4;
  static constexpr uint32_t oInt = oBar + 256;
};

template <int D>
__global__ void __launch_bounds__(NT, 1)
    k_probe_tc(const __nv_bfloat16* __restrict__ Q, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, int N, int Gk, int Gq, int P,
               const int* __restrict__ probe_idx, const int* __restrict__ probe_grp, const int* __restrict__ label_k,
               const unsigned char* __restrict__ route, int keys_per_split, float scale_log2,
               const int* __restrict__ frame_id, const int* __restrict__ fend, int F,
               float* __restrict__ part_o, float* __restrict__ part_ml, int* err) {
  using L = Layout<D>;
  extern __shared__ __align__(1024) unsigned char smem[];
  const uint32_t base = su32(smem);
  if (base & 1023u) {
    if (threadIdx.x == 0) set_error(err, DERR_INDEX);
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * N;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::oBar);
  int* sLab = reinterpret_cast<int*>(smem + L::oLab);
  int* sMisc = reinterpret_cast<int*>(smem + L::oInt);   // [0] tmem, [1] abort
  int* sQrow = sMisc + 8;                                  // [PROWS]
  volatile int* abort_flag = sMisc + 1;

  const int k0 = split * keys_per_split;
  const int k1 = min(N, k0 + keys_per_split);
  const int nchunks = k1 > k0 ? (k1 - k0 + BN - 1) / BN : 0;

  // ---------------- setup ----------------
  for (int r = tid; r < PROWS; r += NT) {
    int row = -1;
    if (r < P) {
      row = probe_idx[(size_t)bh * P + r];
      if (row < 0 || row >= N) { set_error(err, DERR_INDEX); row = -1; }
    }
    sQrow[r] = row;
  }
  if (tid == 0) {
    sMisc[1] = 0;
    mbar_init(su32(&bars->q), 32);
    for (int s = 0; s < 2; ++s) {
      mbar_init(su32(&bars->full[s]), 33);   // 32 label arrivals + the TMA transaction arrival
      mbar_init(su32(&bars->empty[s]), 1 + NSOFT / 32);   // S MMAs done + every softmax warp read the labels
      mbar_init(su32(&bars->vfull[s]), 1);
      mbar_init(su32(&bars->vempty[s]), 1);
      mbar_init(su32(&bars->s_full[s]), 1);
      mbar_init(su32(&bars->s_free[s]), NSOFT / 32);
    }
    mbar_init(su32(&bars->p_full), NSOFT / 32);
    mbar_init(su32(&bars->p_empty), 1);
    mbar_init(su32(&bars->o_done), 1);
    mbar_init(su32(&bars->mma_done), 1);
    mbar_init(su32(&bars->mready[0]), NSOFT / 32);
    mbar_init(su32(&bars->mready[1]), NSOFT / 32);
    mbar_init(su32(&bars->ldone), NSOFT / 32);
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tc_alloc(su32(&sMisc[0]), 512);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = (uint32_t)sMisc[0];
  const uint32_t sQ = base + L::oQ, sK = base + L::oK, sV = base + L::oV;
  const uint32_t tP = tmem + 256, tO = tmem + 384;
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  if (warp == LOAD_WARP) {
    // ---------------- loads ----------------
    constexpr int CPR = D / 8;
    // probe rows, twice (tile rows r and r + 64)
    for (int e = lane; e < BM * CPR; e += 32) {
      const int r = e / CPR, c = e - r * CPR;
      const int row = sQrow[r & (PROWS - 1)];
      cp_async16(sQ + tile_off(r, c, BM), Q + (head + (row < 0 ? 0 : row)) * D + c * 8, row >= 0);
    }
    cp_async_arrive_noinc(su32(&bars->q));
    bool ok = true;
    for (int j = 0; j < nchunks && ok; ++j) {
      const int s = j & 1;
      if (j >= 2) ok = __all_sync(0xffffffffu, wait(bars->empty[s], ((j >> 1) - 1) & 1));
      if (!ok) break;
      const int c0 = k0 + j * BN;
      if (lane == 0) {
        // K rows c0 .. c0+127 of this head (rows past k1 are masked in the softmax)
        mbar_arrive_expect_tx(su32(&bars->full[s]), L::kKV);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_2d(sK + s * L::kKV + h * BN * 128, &tmk, 64 * h, (int)(head + c0), su32(&bars->full[s]));
      }
      for (int r = lane; r < BN; r += 32) {  // 4-byte labels (label rows are only 4-byte aligned)
        const bool v = c0 + r < k1;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(su32(sLab + s * BN + r)),
                     "l"(label_k + head + (v ? c0 + r : 0)), "r"(v ? 4 : 0)
                     : "memory");
      }
      cp_async_arrive_noinc(su32(&bars->full[s]));
      // V rows of the chunk: their stage is free once the PV MMAs two chunks back completed
      if (j >= 2) ok = __all_sync(0xffffffffu, wait(bars->vempty[s], ((j >> 1) - 1) & 1));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(su32(&bars->vfull[s]), L::kKV);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
          tma_load_2d(sV + s * L::kKV + h * BN * 128, &tmv, 64 * h, (int)(head + c0), su32(&bars->vfull[s]));
      }
    }
    cp_async_wait_all();
  } else if (warp == MMA_WARP) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(BM, BN, false);
      constexpr uint32_t IDO = idesc_bf16(BM, D, true);
      bool ok = nchunks == 0 || wait(bars->q, 0);
      auto issue_pv = [&](int i) -> bool {
        if (!wait(bars->p_full, i & 1) || !wait(bars->vfull[i & 1], (i >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t vb = sV + (i & 1) * L::kKV;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t bd = sdesc(vb + k * 2048, (uint32_t)BN * 128, 1024);
          tc_mma_ts(tO, tP + k * 8, bd, IDO, (i > 0 || k > 0) ? 1u : 0u);
          tc_mma_ts(tO, tP + 64 + k * 8, bd, IDO, 1u);
        }
        tc_commit(su32(&bars->vempty[i & 1]));
        tc_commit(su32(&bars->p_empty));
        return true;
      };
      for (int j = 0; ok && j < nchunks; ++j) {
        const int s = j & 1;
        if (!wait(bars->full[s], (j >> 1) & 1)) { ok = false; break; }
        if (j >= 2 && !wait(bars->s_free[s], ((j >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK + s * L::kKV;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t oq = (k >> 2) * (BM * 128) + (k & 3) * 32;
          const uint32_t ok2 = (k >> 2) * (BN * 128) + (k & 3) * 32;
          tc_mma(tmem + s * BN, sdesc(sQ + oq, 16, 1024), sdesc(kb + ok2, 16, 1024), IDS, k > 0 ? 1u : 0u);
        }
        tc_commit(su32(&bars->s_full[s]));
        tc_commit(su32(&bars->empty[s]));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nchunks > 0) issue_pv(nchunks - 1);
      tc_commit(su32(&bars->o_done));
      tc_commit(su32(&bars->mma_done));
      wait(bars->mma_done, 0);
    }
  } else if (warp < 16) {
    // ---------------- softmax (row r, keys of quarter qt) ----------------
    const int qt = warp >> 2, rg = warp & 3;
    const int r = rg * 32 + lane;
    const bool sparse = r >= PROWS;
    const int prow = r & (PROWS - 1);
    const uint32_t lane_off = (uint32_t)(rg * 32) << 16;
    float* xm = reinterpret_cast<float*>(smem + L::oXm);   // [2][4][BM]
    // routed K/V groups of this probe row's query group, as bits (sparse rows only)
    uint32_t rm[4] = {0u, 0u, 0u, 0u};
    if (sparse && prow < P) {
      const int a = probe_grp[(size_t)bh * P + prow];
      if (a >= 0 && a < Gq) {
        const unsigned char* rr = route + ((size_t)bh * Gq + a) * Gk;
        if ((Gk & 15) == 0 && (reinterpret_cast<uintptr_t>(rr) & 15) == 0) {
          uint4 v[8];
#pragma unroll
          for (int c = 0; c < 8; ++c)
            if (c * 16 < Gk) v[c] = __ldg(reinterpret_cast<const uint4*>(rr) + c);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (c * 16 >= Gk) break;
            const uint32_t w4[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if ((w4[q] >> (8 * e)) & 0xffu) rm[c >> 1] |= 1u << ((c & 1) * 16 + q * 4 + e);
          }
        } else {
          for (int g = 0; g < Gk; ++g)
            if (rr[g]) rm[g >> 5] |= 1u << (g & 31);
        }
      }
    }
    // frame-causal: the row sees the keys before fend[its frame] (frame ids nondecreasing)
    int kend = k1;
    if (frame_id && prow < P) {
      const int row = sQrow[prow];
      if (row >= 0) {
        int f = frame_id[row];
        f = f < 0 ? 0 : (f >= F ? F - 1 : f);
        kend = min(k1, fend[f]);
      }
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int b = j & 1;
      // S ready; the chunk's labels (read below) landed before it
      ok = __all_sync(0xffffffffu, wait(bars->s_full[b], (j >> 1) & 1) && wait(bars->full[b], (j >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      const int valid = kend - (k0 + j * BN);
      // keys of this quarter the row may use
      uint32_t km;
      {
        // keys of this quarter before the row's end, then (sparse rows) the routed ones
        const int nv = valid - qt * 32;
        const uint32_t vmask = nv >= 32 ? 0xffffffffu : (nv <= 0 ? 0u : ((1u << nv) - 1u));
        km = vmask;
        if (sparse) {
          const int4* lab4 = reinterpret_cast<const int4*>(sLab + b * BN + qt * 32);
          uint32_t bits = 0u;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int4 g4 = lab4[c];
            const uint32_t gg[4] = {(uint32_t)g4.x, (uint32_t)g4.y, (uint32_t)g4.z, (uint32_t)g4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t g = gg[e];   // a negative label compares as >= Gk
              const uint32_t w01 = (g & 32u) ? rm[1] : rm[0];
              const uint32_t w23 = (g & 32u) ? rm[3] : rm[2];
              const uint32_t w = (g & 64u) ? w23 : w01;
              bits |= ((w >> (g & 31u)) & (g < (uint32_t)Gk ? 1u : 0u)) << (c * 4 + e);
            }
          }
          km &= bits;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(su32(&bars->empty[b]));
      uint32_t sreg[32];
      tc_ld32(tmem + b * BN + lane_off + qt * 32, sreg);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(su32(&bars->s_free[b]));
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if ((km >> e) & 1u) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(sreg[e]));
      xm[(b * 4 + qt) * BM + r] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(su32(&bars->mready[b]));
      ok = __all_sync(0xffffffffu, wait(bars->mready[b], (j >> 1) & 1));
      if (!ok) break;
      float mx = xm[(b * 4 + 0) * BM + r];
#pragma unroll
      for (int q = 1; q < 4; ++q) mx = fmaxf(mx, xm[(b * 4 + q) * BM + r]);
      // every quarter of the row takes the same decision from the same values
      const float mn = fmaxf(m, mx * scale_log2);
      const bool need = (mn > m + kRescaleThreshold) || (m == -INFINITY && mn != -INFINITY);
      const bool warp_need = __any_sync(0xffffffffu, need);
      float alpha = 1.f;
      if (warp_need && mn > m) {
        alpha = (m == -INFINITY) ? 0.f : ex2(m - mn);
        m = mn;
      }
      // P (single buffer) and O are free once PV of the previous chunk has completed
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, wait(bars->p_empty, (j - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        if (warp_need) {
          // this quarter rescales D/4 columns of the row's O
#pragma unroll
          for (int c0 = 0; c0 < D / 4; c0 += 16) {
            uint32_t o[16];
            const uint32_t ta = tO + lane_off + qt * (D / 4) + c0;
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
                "tcgen05.wait::ld.sync.aligned;\n"
                : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]), "=r"(o[7]),
                  "=r"(o[8]), "=r"(o[9]), "=r"(o[10]), "=r"(o[11]), "=r"(o[12]), "=r"(o[13]), "=r"(o[14]), "=r"(o[15])
                : "r"(ta)
                : "memory");
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tc_st16(ta, o);
          }
        }
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t phi[16], plo[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float p0 = ((km >> e) & 1u) ? ex2(__uint_as_float(sreg[e]) * scale_log2 - mu) : 0.f;
        const float p1 = ((km >> (e + 1)) & 1u) ? ex2(__uint_as_float(sreg[e + 1]) * scale_log2 - mu) : 0.f;
        rs[(e >> 1) & 3] += p0 + p1;
        const uint32_t hi = pack_bf16(p0, p1);
        const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&hi);
        phi[e >> 1] = hi;
        plo[e >> 1] = pack_bf16(p0 - __low2float(h2), p1 - __high2float(h2));
      }
      // keys 32 qt .. 32 qt + 31 -> packed columns 16 qt .. 16 qt + 15 of P hi / P lo
      tc_st16(tP + lane_off + 16 * qt, phi);
      tc_st16(tP + lane_off + 64 + 16 * qt, plo);
      tc_fence_before();
      l = l * alpha + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
      __syncwarp();
      if (lane == 0) mbar_arrive(su32(&bars->p_full));
    }
    // ---- this split's outputs: O quarter columns, and (quarter 0) max and the row sum
    float* xl = xm + 2 * 4 * BM;   // [4][BM] partial sums (the maxima buffers may still be read)
    xl[qt * BM + r] = l;
    if (ok && nchunks > 0) ok = __all_sync(0xffffffffu, wait(bars->o_done, 0));
    __syncwarp();
    if (lane == 0) mbar_arrive(su32(&bars->ldone));
    if (ok) ok = __all_sync(0xffffffffu, wait(bars->ldone, 0));
    if (ok) {
      tc_fence_after();
      const size_t rowbase = ((size_t)bh * gridDim.x + split) * PROWS + prow;
      const int acc = sparse ? 1 : 0;
      float* dst = part_o + (rowbase * 2 + acc) * D + qt * (D / 4);
#pragma unroll
      for (int c0 = 0; c0 < D / 4; c0 += 16) {
        uint32_t o[16];
        if (nchunks > 0) {
          const uint32_t ta = tO + lane_off + qt * (D / 4) + c0;
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
              "tcgen05.wait::ld.sync.aligned;\n"
              : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]), "=r"(o[7]),
                "=r"(o[8]), "=r"(o[9]), "=r"(o[10]), "=r"(o[11]), "=r"(o[12]), "=r"(o[13]), "=r"(o[14]), "=r"(o[15])
              : "r"(ta)
              : "memory");
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0u;
        }
        float4* d4 = reinterpret_cast<float4*>(dst + c0);
#pragma unroll
        for (int e = 0; e < 4; ++e)
          d4[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]), __uint_as_float(o[4 * e + 2]),
                              __uint_as_float(o[4 * e + 3]));
      }
      if (qt == 0) {
        part_ml[rowbase * 4 + 2 * acc + 0] = m;
        part_ml[rowbase * 4 + 2 * acc + 1] = (xl[r] + xl[BM + r]) + (xl[2 * BM + r] + xl[3 * BM + r]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == MMA_WARP) tc_dealloc(tmem, 512);
}

}  // namespace ptc

size_t probe_tc_smem_bytes(int D, int Gk) {
  (void)Gk;
  const size_t tiles = D == 64 ? ptc::Layout<64>::oInt : ptc::Layout<128>::oInt;
  const size_t s = tiles + (8 + ptc::PROWS) * 4;
  return s < 120 * 1024 ? 120 * 1024 : s;  // one CTA per SM: it allocates all 512 TMEM columns
}

cudaError_t launch_probe_tc(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk, int Gq, int P,
                            const int* probe_idx, const int* probe_grp, const int* label_k, const unsigned char* route,
                            float scale_log2, int S, const Causal& cz, float* part_o, float* part_ml, int* err,
                            cudaStream_t st) {
  int kps = (N + S - 1) / S;
  kps = (kps + ptc::BN - 1) / ptc::BN * ptc::BN;
  const size_t sm = probe_tc_smem_bytes(D, Gk);
  CUtensorMap tmk, tmv;
  cudaError_t e = make_tmap_bf16_rows(&tmk, K, (unsigned long long)BH * N, D, ptc::BN);
  if (e == cudaSuccess) e = make_tmap_bf16_rows(&tmv, V, (unsigned long long)BH * N, D, ptc::BN);
  if (e != cudaSuccess) return e;
  dim3 grid(S, BH);
  if (D == 64) {
    cudaFuncSetAttribute(ptc::k_probe_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    ptc::k_probe_tc<64><<<grid, ptc::NT, sm, st>>>((const __nv_bfloat16*)Q, tmk, tmv, N, Gk, Gq, P, probe_idx,
                                                   probe_grp, label_k, route, kps, scale_log2, cz.frame_id, cz.fend,
                                                   cz.F, part_o, part_ml, err);
  } else {
    cudaFuncSetAttribute(ptc::k_probe_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    ptc::k_probe_tc<128><<<grid, ptc::NT, sm, st>>>((const __nv_bfloat16*)Q, tmk, tmv, N, Gk, Gq, P, probe_idx,
                                                    probe_grp, label_k, route, kps, scale_log2, cz.frame_id, cz.fend,
                                                    cz.F, part_o, part_ml, err);
  }
  return cudaGetLastError();
}

}  // namespace spr
