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
//               P_j = exp2(S_j * s*log2e - m) in bf16 -> shared memory
//               O  += P_j V_j   (TMEM accumulator, rescaled in place only when a row's
//                                 running max grows by more than 2^8)
// Every mbarrier wait is bounded (2 s); a timeout raises an abort flag that ends every
// role, records DERR_WAIT_TIMEOUT in the workspace and still frees the TMEM.
#include "common.cuh"
#include "kernels.h"

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
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// ---------------------------------------------------------------------------
// PTX wrappers (PTX ISA: mbarrier, cp.async, tcgen05)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;\n" : "=l"(t));
  return t;
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void tc_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t dt, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(dt),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// tcgen05.ld of 32 consecutive 32-bit columns of this warp's 32 lanes, completed
// (tcgen05.wait::ld) inside the same asm statement so no use of r[] can be
// scheduled before the data has landed.
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// tcgen05.ld of 128 consecutive 32-bit columns of this warp's 32 lanes, completed
// (tcgen05.wait::ld) inside the same asm statement so no use of r[] can be
// scheduled before the data has landed.
__device__ __forceinline__ void tc_ld128(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n"
      "tcgen05.wait::ld.sync.aligned;\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}
// tcgen05.st of 32 columns, completed (tcgen05.wait::st) inside the same asm statement.
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n"
      "tcgen05.wait::st.sync.aligned;\n"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm100 format: version 1 at bits
// 46-47, layout type 2 = SWIZZLE_128B at bits 61-63, addresses in 16-byte units).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor of kind::f16: D = f32 (bits 4-5 = 1), A = B = bf16 (bits 7-9,
// 10-12 = 1), A K-major, B K-major (bit 16 = 0) or MN-major (1), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-byte chunk `c` (of the row's D/8 chunks) of row `r` in a tile stored
// as [D/64 halves][rows][64] with 128-byte rows swizzled by (r & 7).
__device__ __forceinline__ uint32_t tile_off(int r, int c, int rows) {
  const int h = c >> 3, cc = c & 7;
  return (uint32_t)(h * rows * 128 + r * 128 + ((cc ^ (r & 7)) << 4));
}

struct Bars {
  uint64_t q, full[2], empty[2], s_full[2], s_free[2], p_full, o_done, mma_done;
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = (uint32_t)D * 128 * 2;  // Q / K / V tile bytes
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oK = oQ + kTile;
  static constexpr uint32_t oV = oK + 2 * kTile;
  static constexpr uint32_t oP = oV + 2 * kTile;
  static constexpr uint32_t oBar = oP + 128 * 128 * 2;
  static constexpr uint32_t oInt = oBar + 256;
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
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  const uint32_t raw = su32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - raw);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const size_t head = (size_t)bh * N;

  Bars* bars = reinterpret_cast<Bars*>(smem + L::oBar);
  int* ints = reinterpret_cast<int*>(smem + L::oInt);
  int* sQrow = ints;                  // [128]
  int* sKrow = sQrow + 128;           // [2][128]
  int* sMisc = sKrow + 256;           // [0] tmem base, [1] abort, [2] total, [3] cnt, [4] slot ok
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
    }
    mbar_init(su32(&bars->p_full), NSOFT);
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
    const uint32_t b = su32(&bar);
    if (mbar_try(b, parity)) return true;
    const uint64_t t0 = gtimer();
    while (true) {
      if (mbar_try(b, parity)) return true;
      if (*abort_flag) return false;
      if (gtimer() - t0 > kTimeoutNs) {
        *abort_flag = 1;
        set_error(err, DERR_WAIT_TIMEOUT);
        return false;
      }
    }
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
      // key row of slot p of chunk j
      {
        const int pos = j * BN + p;
        int row = -1;
        if (pos < total) {
          if (DENSE) {
            row = pos;
          } else {
            int lo = 0, hi = cnt - 1;
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (sCum[mid] <= pos) lo = mid; else hi = mid - 1;
            }
            row = perm_k[head + sKoffL[lo] + (pos - sCum[lo])];
            if (row < 0 || row >= N) { set_error(err, DERR_INDEX); row = -1; }
          }
        }
        sKrow[s * 128 + p] = row;
      }
      named_sync(1, NPROD);
      if (!*prod_ok) break;
      const uint32_t dk = sK + s * L::kTile, dv = sV + s * L::kTile;
      for (int i = 0; i < 32 / RPI; ++i) {
        const int r = pw * 32 + i * RPI + pl / CPR, c = pl % CPR;
        const int row = sKrow[s * 128 + r];
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
        if (!wait(bars->p_full, i & 1)) return false;
        tc_fence_after();
        const uint32_t vb = sV + (i & 1) * L::kTile;
#pragma unroll
        for (int k = 0; k < BN / 16; ++k) {
          const uint64_t ad = sdesc(sP + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc(vb + k * 2048, 16384, 1024);
          tc_mma(tO, ad, bd, IDO, (i > 0 || k > 0) ? 1u : 0u);
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
      if (j >= 1) {
        ok = wait(bars->o_done, (j - 1) & 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (warp_need) {
          // O row *= alpha (in TMEM), warp-uniform
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tc_ld32(tO + lane_off + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tc_st32(tO + lane_off + c * 32, o);
          }
        }
      }
      // P row t -> shared memory ([2 halves][128 rows][64] bf16, 128B-swizzled)
      unsigned char* prow = smem + L::oP;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + tile_off(t, c, 128)) = v;
      }
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(su32(&bars->p_full));
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
  size_t s = 1024 + tiles + (size_t)(128 + 256 + 8 + 3 * Gk + 1) * 4;
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
