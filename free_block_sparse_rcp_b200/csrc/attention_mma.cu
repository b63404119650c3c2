// Route-walking flash attention, warp-level bf16 tensor-core MMA (m16n8k16) with
// fp32 online softmax (gist.science technical summary, section 2.C: attention over
// the routed cells of the group-contiguous layout).
//
// One CTA = one q-tile of up to 128 permuted query rows of one query group (8 warps
// x 16 rows).  Query rows are gathered from their original positions through
// perm_q; the routed key rows of the group are the concatenation, in ascending
// K/V-group order, of the routed groups' permuted segments, gathered from their
// original positions through perm_k in chunks of 64 rows (the permuted layout is
// never materialised).  Slots past the end of the list are masked.  The epilogue
// writes O rows (bf16) and LSE back to the original token positions.
//
// DENSE instantiation: q-tile = 128 consecutive original rows, keys = all rows.
#include "common.cuh"
#include "kernels.h"

namespace spr {
namespace mma {

constexpr int BM = 128;   // query rows per CTA
constexpr int BN = 64;    // key rows per chunk
constexpr int NT = 256;   // threads

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

// byte offset of 16-byte chunk `ch` of row `r` in a [rows][D] bf16 tile (XOR swizzle)
template <int D>
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return (uint32_t)(r * D * 2 + ((ch ^ (r & 7)) << 4));
}

template <int D, bool DENSE>
__global__ void __launch_bounds__(NT, 1)
    k_attn(const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
           const __nv_bfloat16* __restrict__ V, int N, int Gq, int Gk, const int* __restrict__ perm_q,
           const int* __restrict__ perm_k, const int* __restrict__ qoff, const int* __restrict__ koff,
           const int* __restrict__ rlist, const int* __restrict__ rcum, const int* __restrict__ rcnt,
           const int2* __restrict__ tiles, const int* __restrict__ tile_count, int max_tiles,
           float scale_log2, __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int* err) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sQ = smem;                      // [BM][D]
  unsigned char* sK = sQ + BM * D * 2;           // [2][BN][D]
  unsigned char* sV = sK + 2 * BN * D * 2;       // [2][BN][D]
  int* sKrow = reinterpret_cast<int*>(sV + 2 * BN * D * 2);  // [2][BN]
  int* sQrow = sKrow + 2 * BN;                              // [BM]
  int* sList = sQrow + BM;                                  // [Gk] routed groups
  int* sCum = sList + Gk;                                   // [Gk+1]
  int* sKoff = sCum + Gk + 1;                               // [Gk]

  const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t head = (size_t)bh * N;
  int q0, qn, a = 0, total, cnt = 0;
  if (DENSE) {
    q0 = blockIdx.x * BM;
    if (q0 >= N) return;
    qn = min(BM, N - q0);
    total = N;
  } else {
    if ((int)blockIdx.x >= tile_count[bh]) return;
    const int2 tl = tiles[(size_t)bh * max_tiles + blockIdx.x];
    a = tl.x;
    const int* qo = qoff + (size_t)bh * (Gq + 1);
    q0 = qo[a] + tl.y * BM;
    qn = min(BM, qo[a + 1] - q0);
    cnt = rcnt[(size_t)bh * Gq + a];
    const int* rl = rlist + ((size_t)bh * Gq + a) * Gk;
    const int* rc = rcum + ((size_t)bh * Gq + a) * (Gk + 1);
    const int* ko = koff + (size_t)bh * (Gk + 1);
    for (int i = tid; i < cnt; i += NT) {
      sList[i] = rl[i];
      sKoff[i] = ko[rl[i]];
    }
    for (int i = tid; i <= cnt; i += NT) sCum[i] = rc[i];
    total = rc[cnt];
  }
  // query rows
  for (int r = tid; r < BM; r += NT) {
    int row = -1;
    if (r < qn) {
      row = DENSE ? q0 + r : perm_q[head + q0 + r];
      if (row < 0 || row >= N) { set_error(err, DERR_INDEX); row = -1; }
    }
    sQrow[r] = row;
  }
  __syncthreads();
  const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
  for (int e = tid; e < BM * CH; e += NT) {
    int r = e / CH, ch = e - r * CH;
    int row = sQrow[r];
    cp_async16(sQa + swz<D>(r, ch), Q + (head + (row < 0 ? 0 : row)) * D + ch * 8, row >= 0);
  }
  cp_async_commit();

  const int nchunks = (total + BN - 1) / BN;
  auto fill_rows = [&](int j, int buf) {
    for (int s = tid; s < BN; s += NT) {
      int p = j * BN + s, row = -1;
      if (p < total) {
        if (DENSE) {
          row = p;
        } else {
          int lo = 0, hi = cnt - 1;  // largest i with sCum[i] <= p
          while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (sCum[mid] <= p) lo = mid; else hi = mid - 1;
          }
          row = perm_k[head + sKoff[lo] + (p - sCum[lo])];
          if (row < 0 || row >= N) { set_error(err, DERR_INDEX); row = -1; }
        }
      }
      sKrow[buf * BN + s] = row;
    }
  };
  auto issue_kv = [&](int buf) {
    for (int e = tid; e < BN * CH; e += NT) {
      int r = e / CH, ch = e - r * CH;
      int row = sKrow[buf * BN + r];
      const size_t off = (head + (row < 0 ? 0 : row)) * D + ch * 8;
      const uint32_t so = (uint32_t)(buf * BN * D * 2) + swz<D>(r, ch);
      cp_async16(sKa + so, K + off, row >= 0);
      cp_async16(sVa + so, V + off, row >= 0);
    }
    cp_async_commit();
  };
  if (nchunks > 0) {
    fill_rows(0, 0);
    __syncthreads();
    issue_kv(0);
  }

  // per-thread state: rows g = lane/4 and g+8 of the warp's 16-row slice
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  uint32_t qf[D / 16][4];

  cp_async_wait<0>();
  __syncthreads();
  {
    const int r = warp * 16 + (lane & 15);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int ch = kk * 2 + (lane >> 4);
      ldsm_x4(sQa + swz<D>(r, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
    }
  }

  for (int j = 0; j < nchunks; ++j) {
    const int buf = j & 1;
    if (j + 1 < nchunks) {
      fill_rows(j + 1, buf ^ 1);
      __syncthreads();
      issue_kv(buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t kb = sKa + buf * BN * D * 2, vb = sVa + buf * BN * D * 2;
    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[BN / 8][4];
#pragma unroll
    for (int n = 0; n < BN / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < BN / 16; ++np) {
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + swz<D>(key, ch), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kk], b0, b1);
        mma16816(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
    // mask slots past the end of the key list
    const int valid = total - j * BN;
    if (valid < BN) {
#pragma unroll
      for (int n = 0; n < BN / 8; ++n) {
        const int c0 = n * 8 + 2 * (lane & 3);
        if (c0 >= valid) { s[n][0] = -INFINITY; s[n][2] = -INFINITY; }
        if (c0 + 1 >= valid) { s[n][1] = -INFINITY; s[n][3] = -INFINITY; }
      }
    }
    // online softmax (base 2)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mx = -INFINITY;
#pragma unroll
      for (int n = 0; n < BN / 8; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * h], s[n][2 * h + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_r[h], mx * scale_log2);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float corr = ex2(m_r[h] - m_use);
      float sum = 0.f;
#pragma unroll
      for (int n = 0; n < BN / 8; ++n) {
        float p0 = ex2(s[n][2 * h] * scale_log2 - m_use);
        float p1 = ex2(s[n][2 * h + 1] * scale_log2 - m_use);
        s[n][2 * h] = p0;
        s[n][2 * h + 1] = p1;
        sum += p0 + p1;
      }
      l_r[h] = l_r[h] * corr + sum;
      m_r[h] = m_new;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) { o[i][2 * h] *= corr; o[i][2 * h + 1] *= corr; }
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        const int key = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int ch = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + swz<D>(key, ch), b0, b1, b2, b3);
        mma16816(o[2 * dp], pa, b0, b1);
        mma16816(o[2 * dp + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }

  // epilogue: normalise, scatter rows to their original positions
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l = l_r[h];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int r = warp * 16 + (lane >> 2) + 8 * h;
    const int row = sQrow[r];
    if (row < 0) continue;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* orow = O + (head + row) * D;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      const int c = i * 8 + 2 * (lane & 3);
      *reinterpret_cast<uint32_t*>(orow + c) = pack_bf16(o[i][2 * h] * inv, o[i][2 * h + 1] * inv);
    }
    if ((lane & 3) == 0 && lse)
      lse[head + row] = l > 0.f ? (m_r[h] + log2f(l)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace mma

size_t attn_smem_bytes(int D, int Gk) {
  return (size_t)(mma::BM + 4 * mma::BN) * D * 2 + (size_t)(2 * mma::BN + mma::BM + 3 * Gk + 1) * 4;
}

template <int D, bool DENSE>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t st) {
  const size_t sm = attn_smem_bytes(D, DENSE ? 0 : a.Gk);
  auto kern = mma::k_attn<D, DENSE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid(DENSE ? ceil_div(a.N, mma::BM) : a.max_tiles, a.BH);
  kern<<<grid, mma::NT, sm, st>>>((const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.K,
                                  (const __nv_bfloat16*)a.V, a.N, a.Gq, a.Gk, a.perm_q, a.perm_k, a.qoff,
                                  a.koff, a.rlist, a.rcum, a.rcnt, a.tiles, a.tile_count, a.max_tiles,
                                  a.scale_log2, (__nv_bfloat16*)a.O, a.lse, a.err);
  return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs& a, bool dense, cudaStream_t st) {
  if (a.D == 64) return dense ? launch_attn_t<64, true>(a, st) : launch_attn_t<64, false>(a, st);
  return dense ? launch_attn_t<128, true>(a, st) : launch_attn_t<128, false>(a, st);
}

}  // namespace spr
