// Exact probe rows on the tensor cores (gist.science technical summary, section 2.B:
// probe rows evaluated exactly, R = O_dense - O_sparse).
//
// One CTA = the (up to 64) probe rows of one head against one contiguous key split.
// For every 64-key chunk the tensor cores compute S = Q K^T once; the softmax warps
// turn it into two probability tiles -- over all keys (dense) and over the keys whose
// K/V group is routed for the probe row's query group (sparse) -- and the tensor cores
// accumulate both O_dense += P_dense V and O_sparse += P_sparse V in TMEM.  The
// probabilities are kept to ~2^-17 by splitting them into bf16 hi + lo tiles (two MMAs
// each), so the probe outputs carry fp32-level error, not bf16's.  Each split
// writes base-2 running maxima, sums and unnormalised outputs in fp32; the existing
// combine kernel merges the splits.
//
// Roles (256 threads): warps 0-3 softmax (thread t = probe row t, TMEM lane t), warp 4
// TMEM allocation + MMA issue (lane 0), warps 5-7 cp.async loads (probe rows gathered
// through probe_idx; key/value rows and their labels contiguous).  All waits bounded.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace spr {
namespace ptc {

using namespace spr::tc;

constexpr int BM = 128;   // rows of the MMA tile (probe rows + zero padding)
constexpr int BN = 64;    // keys per chunk
constexpr int NSOFT = 128;
constexpr int MMA_WARP = 4;
constexpr int PROD0 = 160;
constexpr int NPROD = 96;
constexpr int NT = 256;
constexpr int PROWS = 64;  // probe rows stored per split (matches the combine's layout)
constexpr float kRescaleThreshold = 8.0f;

struct Bars {
  uint64_t q, full[2], empty[2], s_full[2], s_free[2], p_full, o_done, mma_done;
};

template <int D>
struct Layout {
  static constexpr uint32_t kQ = (uint32_t)BM * D * 2;    // Q tile
  static constexpr uint32_t kKV = (uint32_t)BN * D * 2;   // one K or V chunk
  static constexpr uint32_t kP = (uint32_t)BM * BN * 2;   // one P tile
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kQ;
  static constexpr uint32_t oV = oK + 2 * kKV;
  static constexpr uint32_t oPd = oV + 2 * kKV;            // P_dense hi, then lo at + kP
  static constexpr uint32_t oPs = oPd + 2 * kP;            // P_sparse hi, then lo at + kP
  static constexpr uint32_t oLab = oPs + 2 * kP;           // int [2][BN]
  static constexpr uint32_t oBar = oLab + 2 * BN * 4;
  static constexpr uint32_t oInt = oBar + 256;
};

template <int D>
__global__ void __launch_bounds__(NT, 1)
    k_probe_tc(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
               const __nv_bfloat16* __restrict__ V, int N, int Gk, int Gq, int P, const int* __restrict__ probe_idx,
               const int* __restrict__ probe_grp, const int* __restrict__ label_k,
               const unsigned char* __restrict__ route, int keys_per_split, float scale_log2,
               float* __restrict__ part_o, float* __restrict__ part_ml, int* err) {
  using L = Layout<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = su32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * N;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::oBar);
  int* sLab = reinterpret_cast<int*>(smem + L::oLab);
  int* sMisc = reinterpret_cast<int*>(smem + L::oInt);   // [0] tmem, [1] abort, [2] slot ok
  int* sQrow = sMisc + 8;                                  // [BM]
  unsigned char* sRoute = reinterpret_cast<unsigned char*>(sQrow + BM);  // [BM][Gk]
  volatile int* abort_flag = sMisc + 1;

  const int k0 = split * keys_per_split;
  const int k1 = min(N, k0 + keys_per_split);
  const int nchunks = k1 > k0 ? (k1 - k0 + BN - 1) / BN : 0;

  // ---------------- setup ----------------
  for (int r = tid; r < BM; r += NT) {
    int row = -1;
    if (r < P) {
      row = probe_idx[(size_t)bh * P + r];
      if (row < 0 || row >= N) row = -1;
    }
    sQrow[r] = row;
  }
  for (int e = tid; e < BM * Gk; e += NT) {
    const int r = e / Gk, g = e - r * Gk;
    const int a = r < P ? probe_grp[(size_t)bh * P + r] : -1;
    sRoute[e] = (a >= 0 && a < Gq) ? route[((size_t)bh * Gq + a) * Gk + g] : 0;
  }
  if (tid == 0) {
    sMisc[1] = 0;
    mbar_init(su32(&bars->q), NPROD);
    for (int s = 0; s < 2; ++s) {
      mbar_init(su32(&bars->full[s]), NPROD);
      mbar_init(su32(&bars->empty[s]), 1);
      mbar_init(su32(&bars->s_full[s]), 1);
      mbar_init(su32(&bars->s_free[s]), NSOFT);
    }
    mbar_init(su32(&bars->p_full), NSOFT);
    mbar_init(su32(&bars->o_done), 1);
    mbar_init(su32(&bars->mma_done), 1);
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
  const uint32_t sQ = base + L::oQ, sK = base + L::oK, sV = base + L::oV, sPd = base + L::oPd, sPs = base + L::oPs;
  const uint32_t tS0 = tmem, tOd = tmem + 128, tOs = tmem + 128 + D;   // S buffers at 0 / 64
  auto wait = [&](uint64_t& bar, uint32_t parity) -> bool {
    return bounded_wait(su32(&bar), parity, abort_flag, err);
  };

  if (tid >= PROD0) {
    // ---------------- loads ----------------
    const int p = tid - PROD0;
    constexpr int CPR = D / 8;
    for (int e = p; e < BM * CPR; e += NPROD) {
      const int r = e / CPR, c = e - r * CPR;
      const int row = sQrow[r];
      cp_async16(sQ + tile_off(r, c, BM), Q + (head + (row < 0 ? 0 : row)) * D + c * 8, row >= 0);
    }
    cp_async_arrive_noinc(su32(&bars->q));
    volatile int* prod_ok = sMisc + 2;
    for (int j = 0; j < nchunks; ++j) {
      const int s = j & 1;
      if (p == 0) *prod_ok = (j < 2 || wait(bars->empty[s], ((j >> 1) - 1) & 1)) ? 1 : 0;
      named_sync(1, NPROD);
      if (!*prod_ok) break;
      const int c0 = k0 + j * BN;
      const uint32_t dk = sK + s * L::kKV, dv = sV + s * L::kKV;
      // 64 rows x CPR chunks for K and for V: 2 * 64 * CPR / 128 per thread
      for (int e = p; e < BN * CPR; e += NPROD) {
        const int r = e / CPR, c = e - r * CPR;
        const bool ok = c0 + r < k1;
        const size_t off = (head + (ok ? c0 + r : 0)) * D + c * 8;
        const uint32_t o = tile_off(r, c, BN);
        cp_async16(dk + o, K + off, ok);
        cp_async16(dv + o, V + off, ok);
      }
      for (int r = p; r < BN; r += NPROD) {  // 4-byte labels (label rows are only 4-byte aligned)
        const bool v = c0 + r < k1;
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(su32(sLab + s * BN + r)),
                     "l"(label_k + head + (v ? c0 + r : 0)), "r"(v ? 4 : 0)
                     : "memory");
      }
      cp_async_arrive_noinc(su32(&bars->full[s]));
    }
    cp_async_wait_all();
  } else if (warp == MMA_WARP) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t IDS = idesc_bf16(BM, BN, false);
      constexpr uint32_t IDO = idesc_bf16(BM, D, true);
      bool ok = nchunks == 0 || wait(bars->q, 0);
      auto issue_pv = [&](int i) -> bool {
        if (!wait(bars->p_full, i & 1)) return false;
        tc_fence_after();
        const uint32_t vb = sV + (i & 1) * L::kKV;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t bd = sdesc(vb + k * 2048, (uint32_t)BN * 128, 1024);
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          tc_mma(tOd, sdesc(sPd + k * 32, 16, 1024), bd, IDO, acc);
          tc_mma(tOd, sdesc(sPd + L::kP + k * 32, 16, 1024), bd, IDO, 1u);
          tc_mma(tOs, sdesc(sPs + k * 32, 16, 1024), bd, IDO, acc);
          tc_mma(tOs, sdesc(sPs + L::kP + k * 32, 16, 1024), bd, IDO, 1u);
        }
        tc_commit(su32(&bars->empty[i & 1]));
        tc_commit(su32(&bars->o_done));
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
          tc_mma(tS0 + s * BN, sdesc(sQ + oq, 16, 1024), sdesc(kb + ok2, 16, 1024), IDS, k > 0 ? 1u : 0u);
        }
        tc_commit(su32(&bars->s_full[s]));
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nchunks > 0) issue_pv(nchunks - 1);
      tc_commit(su32(&bars->mma_done));
      wait(bars->mma_done, 0);
    }
  } else {
    // ---------------- softmax (thread t = row t) ----------------
    const int t = tid;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const unsigned char* rrow = sRoute + t * Gk;
    float md = -INFINITY, ld = 0.f, ms = -INFINITY, ls = 0.f;
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, wait(bars->s_full[b], (j >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[64];
      tc_ld32(tS0 + lane_off + b * BN, sr);
      tc_ld32(tS0 + lane_off + b * BN + 32, sr + 32);
      tc_fence_before();
      mbar_arrive(su32(&bars->s_free[b]));
      const int valid = k1 - (k0 + j * BN);
      const int* lab = sLab + b * BN;
      uint64_t rmask = 0;  // bit c: key c is routed for this row
      float mxd = -INFINITY, mxs = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c) {
        if (c < valid) {
          const float x = __uint_as_float(sr[c]);
          mxd = fmaxf(mxd, x);
          const int g = lab[c];
          if (g >= 0 && g < Gk && rrow[g]) {
            rmask |= 1ull << c;
            mxs = fmaxf(mxs, x);
          }
        }
      }
      const float mnd = fmaxf(md, mxd * scale_log2);
      const float mns = fmaxf(ms, mxs * scale_log2);
      const bool need = (mnd > md + kRescaleThreshold) || (mns > ms + kRescaleThreshold) ||
                        (md == -INFINITY && mnd != -INFINITY) || (ms == -INFINITY && mns != -INFINITY);
      const bool warp_need = __any_sync(0xffffffffu, need);
      float ad = 1.f, as = 1.f;
      if (warp_need) {
        if (mnd > md) { ad = (md == -INFINITY) ? 0.f : ex2(md - mnd); md = mnd; }
        if (mns > ms) { as = (ms == -INFINITY) ? 0.f : ex2(ms - mns); ms = mns; }
      }
      const float mud = md == -INFINITY ? 0.f : md, mus = ms == -INFINITY ? 0.f : ms;
      uint32_t pd[BN / 2], ps[BN / 2], pdl[BN / 2], psl[BN / 2];
      float sd = 0.f, ss = 0.f;
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        float e0 = 0.f, e1 = 0.f, f0 = 0.f, f1 = 0.f;
        if (c < valid) {
          const float x = __uint_as_float(sr[c]) * scale_log2;
          e0 = ex2(x - mud);
          if ((rmask >> c) & 1) f0 = ex2(x - mus);
        }
        if (c + 1 < valid) {
          const float x = __uint_as_float(sr[c + 1]) * scale_log2;
          e1 = ex2(x - mud);
          if ((rmask >> (c + 1)) & 1) f1 = ex2(x - mus);
        }
        sd += e0 + e1;
        ss += f0 + f1;
        pd[c >> 1] = pack_bf16(e0, e1);
        ps[c >> 1] = pack_bf16(f0, f1);
        const __nv_bfloat162 hd = *reinterpret_cast<const __nv_bfloat162*>(&pd[c >> 1]);
        const __nv_bfloat162 hs = *reinterpret_cast<const __nv_bfloat162*>(&ps[c >> 1]);
        pdl[c >> 1] = pack_bf16(e0 - __low2float(hd), e1 - __high2float(hd));
        psl[c >> 1] = pack_bf16(f0 - __low2float(hs), f1 - __high2float(hs));
      }
      ld = ld * ad + sd;
      ls = ls * as + ss;
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, wait(bars->o_done, (j - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        if (warp_need) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc_ld32(tOd + lane_off + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * ad);
            tc_st32(tOd + lane_off + c * 32, o);
            tc_ld32(tOs + lane_off + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * as);
            tc_st32(tOs + lane_off + c * 32, o);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < BN / 8; ++c) {
        const uint32_t o = tile_off(t, c, BM);
        *reinterpret_cast<uint4*>(smem + L::oPd + o) = make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
        *reinterpret_cast<uint4*>(smem + L::oPd + L::kP + o) =
            make_uint4(pdl[4 * c], pdl[4 * c + 1], pdl[4 * c + 2], pdl[4 * c + 3]);
        *reinterpret_cast<uint4*>(smem + L::oPs + o) = make_uint4(ps[4 * c], ps[4 * c + 1], ps[4 * c + 2], ps[4 * c + 3]);
        *reinterpret_cast<uint4*>(smem + L::oPs + L::kP + o) =
            make_uint4(psl[4 * c], psl[4 * c + 1], psl[4 * c + 2], psl[4 * c + 3]);
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(su32(&bars->p_full));
    }
    if (ok && nchunks > 0) ok = __all_sync(0xffffffffu, wait(bars->o_done, (nchunks - 1) & 1));
    if (ok) {
      tc_fence_after();
      const size_t rowbase = ((size_t)bh * gridDim.x + split) * PROWS + t;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t od[32], os[32];
        if (nchunks > 0) {
          tc_ld32(tOd + lane_off + c * 32, od);
          tc_ld32(tOs + lane_off + c * 32, os);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) od[e] = os[e] = 0u;
        }
        if (t < PROWS) {
          float4* dd = reinterpret_cast<float4*>(part_o + (rowbase * 2 + 0) * D + c * 32);
          float4* dsp = reinterpret_cast<float4*>(part_o + (rowbase * 2 + 1) * D + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            dd[e] = make_float4(__uint_as_float(od[4 * e]), __uint_as_float(od[4 * e + 1]),
                                __uint_as_float(od[4 * e + 2]), __uint_as_float(od[4 * e + 3]));
            dsp[e] = make_float4(__uint_as_float(os[4 * e]), __uint_as_float(os[4 * e + 1]),
                                 __uint_as_float(os[4 * e + 2]), __uint_as_float(os[4 * e + 3]));
          }
        }
      }
      if (t < PROWS) {
        part_ml[rowbase * 4 + 0] = md;
        part_ml[rowbase * 4 + 1] = ld;
        part_ml[rowbase * 4 + 2] = ms;
        part_ml[rowbase * 4 + 3] = ls;
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
  const size_t tiles = D == 64 ? ptc::Layout<64>::oInt : ptc::Layout<128>::oInt;
  const size_t s = 1024 + tiles + (8 + ptc::BM) * 4 + (size_t)ptc::BM * Gk;
  return s < 120 * 1024 ? 120 * 1024 : s;  // one CTA per SM: it allocates all 512 TMEM columns
}

cudaError_t launch_probe_tc(const void* Q, const void* K, const void* V, int BH, int N, int D, int Gk, int Gq, int P,
                            const int* probe_idx, const int* probe_grp, const int* label_k, const unsigned char* route,
                            float scale_log2, int S, float* part_o, float* part_ml, int* err, cudaStream_t st) {
  int kps = (N + S - 1) / S;
  kps = (kps + ptc::BN - 1) / ptc::BN * ptc::BN;
  const size_t sm = probe_tc_smem_bytes(D, Gk);
  dim3 grid(S, BH);
  if (D == 64) {
    cudaFuncSetAttribute(ptc::k_probe_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    ptc::k_probe_tc<64><<<grid, ptc::NT, sm, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                                   (const __nv_bfloat16*)V, N, Gk, Gq, P, probe_idx, probe_grp,
                                                   label_k, route, kps, scale_log2, part_o, part_ml, err);
  } else {
    cudaFuncSetAttribute(ptc::k_probe_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    ptc::k_probe_tc<128><<<grid, ptc::NT, sm, st>>>((const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                                    (const __nv_bfloat16*)V, N, Gk, Gq, P, probe_idx, probe_grp,
                                                    label_k, route, kps, scale_log2, part_o, part_ml, err);
  }
  return cudaGetLastError();
}

}  // namespace spr
