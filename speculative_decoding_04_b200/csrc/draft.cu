// Markov-head draft stage: gamma serial steps of
//   l_d = U_k + W1[x_{k-1}] · W2 ;  x_k ~ softmax(l_d / T)   (argmax when T == 0)
// [P3 "DSpark Speculative Decoding" §Semi-Autoregressive Generation: p_k(v) ∝ exp(U_k(v) + B_k(v)),
//  B(x_{k-1}, ·) = W1[x_{k-1}] W2 of low rank r]
// [P1 "DeepSeek V4-Pro DSpark 推测解码方案深度解析" §DSpark 架构设计：半自回归生成与马尔可夫修正:
//  the sequential head only looks at the previous sampled token, position by position]
//
// Each step is two kernels chained by programmatic dependent launch:
//   main pass  -- bias contraction fused with U + bias, the l_d store and per-(request,
//                 32-column chunk) softmax statistics (max, sum of exp) or greedy top-2.
//                 Two variants: a CUDA-core GEMV for few requests (or fp32 weights) and a
//                 tcgen05 tensor-core GEMM with TMA-staged W2 / U / l_d tiles.
//   combine    -- per request: global max and normaliser from the chunk statistics (fp64),
//                 exclusive scan to the chunk that crosses u * S, exact rescan of that one
//                 chunk, x_k and the near-tie flag.
// The main pass of step k+1 prefetches its W2 / U tiles before waiting on step k's combine.

#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dspark {

constexpr int kChunk = 32;

struct DraftArgs {
  const float* U;
  const void* W1;
  const void* W2;
  const int32_t* x0;
  int32_t* x_out;
  float* ld;
  const float* u_draft;
  uint32_t* flags;
  ChunkStat* part;
  uint32_t* status;
  int B, gamma, V, r, nchunk;
  float inv_T;
  int greedy;
};

// exp(z - m) as 2^((z - m) log2 e); z and m are already-rounded fp32 values
__device__ __forceinline__ float ex_shift(float z, float m) { return exp2f(__fmul_rn(__fsub_rn(z, m), kLog2e)); }

__device__ __forceinline__ int prev_token(const DraftArgs& a, int b, int k, bool report) {
  int prev = (k == 0) ? a.x0[b] : a.x_out[b * a.gamma + k - 1];
  if ((unsigned)prev >= (unsigned)a.V) {
    if (report) atomicOr(a.flags + b, DSPARK_FLAG_TOKEN_RANGE);
    prev = prev < 0 ? 0 : a.V - 1;
  }
  return prev;
}

// ============================================================================ CUDA-core GEMV main pass

template <typename WT>
__device__ __forceinline__ float wload(const void* p, size_t i);
template <>
__device__ __forceinline__ float wload<float>(const void* p, size_t i) {
  return static_cast<const float*>(p)[i];
}
template <>
__device__ __forceinline__ float wload<__nv_bfloat16>(const void* p, size_t i) {
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

template <typename WT>
__device__ __forceinline__ void wload8(const void* p, size_t off, float (&w)[8]);
template <>
__device__ __forceinline__ void wload8<float>(const void* p, size_t off, float (&w)[8]) {
  const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + off);
  float4 x = __ldg(q), y = __ldg(q + 1);
  w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
  w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
}
template <>
__device__ __forceinline__ void wload8<__nv_bfloat16>(const void* p, size_t off, float (&w)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + off));
  const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[2 * i] = __uint_as_float(q[i] << 16);
    w[2 * i + 1] = __uint_as_float(q[i] & 0xFFFF0000u);
  }
}

// Chunk statistics over 16 lanes x 2 columns (one 32-column chunk per half-warp).
__device__ __forceinline__ ChunkStat chunk_stat_pair(float l0, float l1, bool val0, bool val1, int v,
                                                     float inv_T, int greedy) {
  ChunkStat st;
  if (greedy) {
    Top2 t;
    t.best = val0 ? l0 : -INFINITY;
    t.idx = val0 ? v : -1;
    t.second = -INFINITY;
    Top2 u;
    u.best = val1 ? l1 : -INFINITY;
    u.idx = val1 ? v + 1 : -1;
    u.second = -INFINITY;
    t = top2_merge(t, u);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) t = top2_merge(t, top2_shfl_xor(t, o));
    st.m = t.best;
    st.s = 0.f;
    st.idx = t.idx;
    st.m2 = t.second;
  } else {
    const float z0 = val0 ? __fmul_rn(l0, inv_T) : -INFINITY;
    const float z1 = val1 ? __fmul_rn(l1, inv_T) : -INFINITY;
    float m = fmaxf(z0, z1);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = (val0 ? ex_shift(z0, m) : 0.f) + (val1 ? ex_shift(z1, m) : 0.f);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    st.m = m;
    st.s = s;
    st.idx = 0;
    st.m2 = 0.f;
  }
  return st;
}

// Grid: x = 256-column tile, y = group of BG requests.  128 threads: the r rank-dimension is
// split over the 4 warps, each lane owns 8 consecutive columns; the partial sums meet in
// shared memory, then every thread finishes 2 columns for each request of the group.
template <typename WT, int BG>
__global__ void __launch_bounds__(128) draft_main_fma(DraftArgs a, int k, int vec_ok) {
  extern __shared__ __align__(16) float fsm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int v0 = blockIdx.x * 256;
  const int b0 = blockIdx.y * BG;
  const int nb = min(BG, a.B - b0);
  const int r = a.r, V = a.V;
  float* G = fsm;                                          // [BG][r]
  float* red = fsm + ((BG * r + 3) & ~3);                   // [4][BG][256]

  pdl_trigger();
  pdl_wait();
  for (int i = tid; i < BG * r; i += blockDim.x) {
    const int bb = i / r, kk = i - bb * r;
    float g = 0.f;
    if (bb < nb) g = wload<WT>(a.W1, (size_t)prev_token(a, b0 + bb, k, kk == 0) * r + kk);
    G[i] = g;
  }
  __syncthreads();

  const int kper = (r + 3) / 4;
  const int kbeg = min(r, warp * kper), kend = min(r, kbeg + kper);
  const int vl = v0 + lane * 8;
  float acc[BG][8];
#pragma unroll
  for (int bb = 0; bb < BG; ++bb)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[bb][j] = 0.f;
  if (vec_ok && vl + 8 <= V) {
#pragma unroll 4
    for (int kk = kbeg; kk < kend; ++kk) {
      float w[8];
      wload8<WT>(a.W2, (size_t)kk * V + vl, w);
#pragma unroll
      for (int bb = 0; bb < BG; ++bb) {
        const float g = G[bb * r + kk];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[bb][j] = fmaf(g, w[j], acc[bb][j]);
      }
    }
  } else {
    for (int kk = kbeg; kk < kend; ++kk) {
      float w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) w[j] = (vl + j < V) ? wload<WT>(a.W2, (size_t)kk * V + vl + j) : 0.f;
#pragma unroll
      for (int bb = 0; bb < BG; ++bb) {
        const float g = G[bb * r + kk];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[bb][j] = fmaf(g, w[j], acc[bb][j]);
      }
    }
  }
#pragma unroll
  for (int bb = 0; bb < BG; ++bb)
#pragma unroll
    for (int j = 0; j < 8; ++j) red[(warp * BG + bb) * 256 + lane * 8 + j] = acc[bb][j];
  __syncthreads();

  const int c = 2 * tid;
  const int v = v0 + c;
  const bool val0 = v < V, val1 = v + 1 < V;
  const int chunk = v0 / kChunk + (tid >> 4);
  for (int bb = 0; bb < nb; ++bb) {
    const int b = b0 + bb;
    float bias0 = 0.f, bias1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      bias0 += red[(w * BG + bb) * 256 + c];
      bias1 += red[(w * BG + bb) * 256 + c + 1];
    }
    const size_t row = ((size_t)b * a.gamma + k) * V;
    float l0 = 0.f, l1 = 0.f;
    if (val0) {
      l0 = a.U[row + v] + bias0;
      a.ld[row + v] = l0;
    }
    if (val1) {
      l1 = a.U[row + v + 1] + bias1;
      a.ld[row + v + 1] = l1;
    }
    if ((val0 && !isfinite(l0)) || (val1 && !isfinite(l1))) atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
    const ChunkStat st = chunk_stat_pair(l0, l1, val0, val1, v, a.inv_T, a.greedy);
    if ((tid & 15) == 0 && chunk < a.nchunk) a.part[(size_t)b * a.nchunk + chunk] = st;
  }
}

// ============================================================================ tcgen05 main pass
//
// One CTA per SM: a group of up to 128 requests (MMA M = 128, row = request) times a
// contiguous run of 64-column tiles (MMA N = 64, K = r).  Warp roles:
//   warp 0      TMA producer: W2 tile [r x 64] bf16 (MN-major, 128B swizzle) and the two
//               U boxes [rows x 32] fp32 of the tile, 3 / 2 stage rings.
//   warp 1      MMA issuer: r/16 tcgen05.mma kind::f16 per tile into one of two TMEM
//               accumulators (64 fp32 columns each).
//   warp 2      TMEM allocation owner.
//   warps 4-11  epilogue, two warpgroups (columns 0-31 / 32-63 of each tile): thread = request
//               row; TMEM -> registers, + U from the swizzled smem box, l_d written back to the
//               box and stored by TMA, chunk statistics from registers.
// A (the gathered W1 rows, K-major, 128B swizzle) is built once per step by warps 1-11.

constexpr int kTcN = 64;
constexpr int kTcStagesW = 3;
constexpr int kTcStagesU = 2;
constexpr int kTcThreads = 384;
constexpr uint32_t kTcTmemCols = 128;

struct TcLayout {
  uint32_t g, w2, u, bars, misc, total;
  uint32_t w2_stage_bytes, u_box_bytes;
};

__host__ __device__ inline TcLayout tc_layout(int r, int box_rows) {
  TcLayout L;
  L.g = 0;
  L.w2_stage_bytes = (uint32_t)r * 128u;
  L.w2 = L.g + (uint32_t)(r / 64) * 16384u;
  L.u_box_bytes = (uint32_t)box_rows * 128u;
  L.u = L.w2 + kTcStagesW * L.w2_stage_bytes;
  L.bars = L.u + kTcStagesU * 2 * L.u_box_bytes;
  L.misc = L.bars + 8u * (2 * kTcStagesW + 2 * kTcStagesU + 2 + 2 + 1);
  L.total = L.misc + 16u;
  return L;
}

struct TcSync {
  volatile int* abort;
  uint32_t* status;
};

// Bounded mbarrier wait shared by all roles; after any timeout every later wait returns at once.
__device__ __forceinline__ bool tc_wait(const TcSync& s, uint64_t* bar, uint32_t parity) {
  if (*s.abort) return false;
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *s.abort) return false;
  }
  *s.abort = 1;
  atomicOr(s.status, (uint32_t)DSPARK_ETIMEOUT);
  return false;
}

__global__ void __launch_bounds__(kTcThreads, 1)
    draft_main_tc(const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmU,
                  const __grid_constant__ CUtensorMap tmLD, DraftArgs a, int k, int ntiles, int n_bgroups,
                  int ctas_per_group, int box_rows) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const TcLayout L = tc_layout(a.r, box_rows);
  uint8_t* sG = sm + L.g;
  uint8_t* sW = sm + L.w2;
  uint8_t* sU = sm + L.u;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* w_full = bars;
  uint64_t* w_empty = w_full + kTcStagesW;
  uint64_t* u_full = w_empty + kTcStagesW;
  uint64_t* u_empty = u_full + kTcStagesU;
  uint64_t* t_full = u_empty + kTcStagesU;
  uint64_t* t_empty = t_full + 2;
  uint64_t* mma_done = t_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L.misc + 4);
  const TcSync sy{s_abort, a.status};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % n_bgroups;
  const int jc = blockIdx.x / n_bgroups;
  const int t_beg = (int)((long long)jc * ntiles / ctas_per_group);
  const int t_end = (int)((long long)(jc + 1) * ntiles / ctas_per_group);
  const int nt = t_end - t_beg;
  const int b0 = g * 128;
  const int ksteps = a.r / 16;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStagesW; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], 1);
    }
    for (int i = 0; i < kTcStagesU; ++i) {
      mbar_init(&u_full[i], 1);
      mbar_init(&u_empty[i], 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&t_full[i], 1);
      mbar_init(&t_empty[i], 8);
    }
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmW2);
    prefetch_tmap(&tmU);
    prefetch_tmap(&tmLD);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // W2 and U are inputs of the call, so the ring fills before the previous kernel finishes.
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int v0 = (t_beg + i) * kTcN;
        const int s = i % kTcStagesW, su = i % kTcStagesU;
        if (!tc_wait(sy, &w_empty[s], ((i / kTcStagesW) & 1) ^ 1)) break;
        mbar_arrive_expect_tx(&w_full[s], L.w2_stage_bytes);
        tma_load_2d(sW + s * L.w2_stage_bytes, &tmW2, v0, 0, &w_full[s]);
        if (!tc_wait(sy, &u_empty[su], ((i / kTcStagesU) & 1) ^ 1)) {
          issued = i + 1;
          break;
        }
        uint8_t* ub = sU + su * 2 * L.u_box_bytes;
        mbar_arrive_expect_tx(&u_full[su], 2 * L.u_box_bytes);
        tma_load_3d(ub, &tmU, v0, k, b0, &u_full[su]);
        tma_load_3d(ub + L.u_box_bytes, &tmU, v0 + 32, k, b0, &u_full[su]);
        issued = i + 1;
      }
      if (*s_abort) {
        // give the copies already issued a bounded chance to land before the CTA exits
        for (int i = max(0, issued - kTcStagesW); i < issued; ++i)
          for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(&w_full[i % kTcStagesW], (i / kTcStagesW) & 1); ++t) {
          }
      }
    }
  } else {
    pdl_wait();
    // ---------------------------------------------------------------- gather A = W1[x_{k-1}] rows
    {
      const int cpr = a.r / 8;  // 16-byte chunks per row
      const __nv_bfloat16* W1 = static_cast<const __nv_bfloat16*>(a.W1);
      for (int i = threadIdx.x - 32; i < 128 * cpr; i += kTcThreads - 32) {
        const int row = i / cpr, c = i - row * cpr;
        const int b = b0 + row;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (b < a.B) val = __ldg(reinterpret_cast<const uint4*>(W1 + (size_t)prev_token(a, b, k, c == 0) * a.r + c * 8));
        const int kb = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(sG + kb * 16384 + row * 128 + ((cc ^ (row & 7)) << 4)) = val;
      }
      fence_proxy_async_smem();
      named_bar(1, kTcThreads - 32);
    }
    if (warp == 1) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t idesc = (1u << 4)                        // D fp32
                               | (1u << 7) | (1u << 10)         // A, B bf16
                               | (1u << 16)                     // B MN-major (W2 is [r][V])
                               | ((uint32_t)(kTcN >> 3) << 17)  // N
                               | ((uint32_t)(128 >> 4) << 24);  // M
        const uint32_t g_addr = smem_u32(sG), w_addr = smem_u32(sW);
        for (int i = 0; i < nt; ++i) {
          const int acc = i & 1, s = i % kTcStagesW;
          if (!tc_wait(sy, &t_empty[acc], ((i >> 1) & 1) ^ 1)) break;
          if (!tc_wait(sy, &w_full[s], (i / kTcStagesW) & 1)) break;
          tc_fence_after();
          const uint32_t wst = w_addr + s * L.w2_stage_bytes;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint64_t ad = smem_desc(g_addr + (kk >> 2) * 16384u + (kk & 3) * 32u, 16u, 1024u, 2u);
            const uint64_t bd = smem_desc(wst + kk * 2048u, L.w2_stage_bytes, 1024u, 2u);
            tc_mma_f16(tmem_base + acc * kTcN, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(&w_empty[s]);
          tc_commit(&t_full[acc]);
        }
        tc_commit(mma_done);
      }
      __syncwarp();
    } else if (warp >= 4) {
      // ---------------------------------------------------------------- epilogue
      const int ew = warp - 4, h = ew >> 2, q = ew & 3;
      const int row = q * 32 + lane;
      const int b = b0 + row;
      const bool live = (b < a.B) && (row < box_rows);
      bool bad = false;
      for (int i = 0; i < nt; ++i) {
        const int v0 = (t_beg + i) * kTcN;
        const int acc = i & 1, su = i % kTcStagesU;
        const int vb = v0 + h * 32;
        float bias[32];
        const bool ok_t = tc_wait(sy, &t_full[acc], (i >> 1) & 1);
        const bool all_t = __all_sync(0xffffffffu, ok_t);
        if (all_t) {
          tc_fence_after();
          tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * kTcN + h * 32, bias);
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&t_empty[acc]);
        const bool ok_u = tc_wait(sy, &u_full[su], (i / kTcStagesU) & 1);
        uint8_t* ubox = sU + su * 2 * L.u_box_bytes + h * L.u_box_bytes;
        if (live && all_t && ok_u) {
          uint8_t* rp = ubox + row * 128;
          float l[32];
#pragma unroll
          for (int j8 = 0; j8 < 8; ++j8) {
            float4* p = reinterpret_cast<float4*>(rp + ((j8 ^ (row & 7)) << 4));
            float4 u4 = *p;
            u4.x += bias[4 * j8 + 0];
            u4.y += bias[4 * j8 + 1];
            u4.z += bias[4 * j8 + 2];
            u4.w += bias[4 * j8 + 3];
            *p = u4;
            l[4 * j8 + 0] = u4.x;
            l[4 * j8 + 1] = u4.y;
            l[4 * j8 + 2] = u4.z;
            l[4 * j8 + 3] = u4.w;
          }
          const int nvalid = min(32, a.V - vb);
          ChunkStat st;
          if (a.greedy) {
            Top2 t;
            t.best = -INFINITY;
            t.idx = -1;
            t.second = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nvalid) {
                bad |= !isfinite(l[j]);
                const float x = l[j];
                if (t.idx < 0 || x > t.best) {
                  t.second = fmaxf(t.second, t.best);
                  t.best = x;
                  t.idx = vb + j;
                } else {
                  t.second = fmaxf(t.second, x);
                }
              }
            }
            st.m = t.best;
            st.s = 0.f;
            st.idx = t.idx;
            st.m2 = t.second;
          } else {
            float z[32];
            float m = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              z[j] = __fmul_rn(l[j], a.inv_T);
              if (j < nvalid) {
                bad |= !isfinite(l[j]);
                m = fmaxf(m, z[j]);
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) z[j] = (j < nvalid) ? ex_shift(z[j], m) : 0.f;
#pragma unroll
            for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
              for (int j = 0; j < w; ++j) z[j] += z[j + w];
            st.m = m;
            st.s = z[0];
            st.idx = 0;
            st.m2 = 0.f;
          }
          if (vb < a.V) a.part[(size_t)b * a.nchunk + vb / kChunk] = st;
        }
        fence_proxy_async_smem();
        named_bar(2 + h, 128);
        if (q == 0 && lane == 0) {
          if (vb < a.V && ok_u && !*s_abort) {
            tma_store_3d(&tmLD, ubox, vb, k, b0);
            bulk_commit();
            bulk_wait_read0();
          }
          mbar_arrive(&u_empty[su]);
        }
      }
      if (q == 0 && lane == 0) bulk_wait0();
      if (bad) atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
    }
  }
  __syncthreads();
  if (warp == 2) {
    // every MMA issued has to finish before the columns are released
    for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(mma_done, 0); ++t) {
    }
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
  if (threadIdx.x == 0 && *s_abort && a.flags)
    for (int i = 0; i < min(128, a.B - b0); ++i) atomicOr(a.flags + b0 + i, DSPARK_FLAG_DEVICE_TIMEOUT);
}

// ============================================================================ combine + sample

// One CTA per request.  Softmax: load the chunk (max, sum) pairs, global max M, per-thread
// fp64 sums over contiguous chunk ranges, block scan, the crossing thread walks its chunks to
// the chunk holding u*S, and one warp rescans that chunk's 32 stored logits in fp64.
constexpr int kCombThreads = 256;

__global__ void __launch_bounds__(kCombThreads) draft_combine(DraftArgs a, int k) {
  extern __shared__ __align__(16) float csm[];
  __shared__ double s_warp[kCombThreads / 32];
  __shared__ float s_wmax[kCombThreads / 32];
  __shared__ Top2 s_top[kCombThreads / 32];
  __shared__ int s_chunk;
  __shared__ double s_base, s_S, s_t;
  __shared__ float s_M;
  const int b = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nchunk = a.nchunk;
  const ChunkStat* P = a.part + (size_t)b * nchunk;
  pdl_trigger();
  pdl_wait();

  if (a.greedy) {
    Top2 t;
    t.best = -INFINITY;
    t.idx = -1;
    t.second = -INFINITY;
    for (int c = tid; c < nchunk; c += kCombThreads) {
      const ChunkStat s = P[c];
      Top2 u;
      u.best = s.m;
      u.idx = s.idx;
      u.second = s.m2;
      t = top2_merge(t, u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t = top2_merge(t, top2_shfl_xor(t, o));
    if (lane == 0) s_top[warp] = t;
    __syncthreads();
    if (tid == 0) {
      Top2 r = s_top[0];
      for (int w = 1; w < kCombThreads / 32; ++w) r = top2_merge(r, s_top[w]);
      int x = r.idx;
      if (x < 0 || x >= a.V) {
        atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
        x = min(max(x, 0), a.V - 1);
      }
      if (r.best - r.second <= 1e-6f * fmaxf(1.f, fabsf(r.best))) atomicOr(a.flags + b, DSPARK_FLAG_DRAFT_NEAR_TIE);
      a.x_out[b * a.gamma + k] = x;
    }
    return;
  }

  float* sm_m = csm;           // [nchunk]
  float* sm_s = csm + nchunk;  // [nchunk]
  float mloc = -INFINITY;
  for (int c = tid; c < nchunk; c += kCombThreads) {
    const float2 ms = *reinterpret_cast<const float2*>(P + c);
    sm_m[c] = ms.x;
    sm_s[c] = ms.y;
    mloc = fmaxf(mloc, ms.x);
  }
  mloc = warp_max(mloc);
  if (lane == 0) s_wmax[warp] = mloc;
  __syncthreads();
  if (tid == 0) {
    float M = s_wmax[0];
    for (int w = 1; w < kCombThreads / 32; ++w) M = fmaxf(M, s_wmax[w]);
    s_M = M;
  }
  __syncthreads();
  const float M = s_M;
  const double Md = (double)M;

  // contiguous chunk range of this thread
  const int per = (nchunk + kCombThreads - 1) / kCombThreads;
  const int c0 = min(nchunk, tid * per), c1 = min(nchunk, c0 + per);
  double tsum = 0.0;
  for (int c = c0; c < c1; ++c) tsum += (double)sm_s[c] * exp((double)sm_m[c] - Md);
  // block exclusive scan of tsum (fp64); [pre, nxt) of consecutive threads tile [0, S) exactly
  const double incl = warp_incl_scan_d(tsum);
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  double wpre = 0.0;
  for (int w = 0; w < warp; ++w) wpre += s_warp[w];
  double S = 0.0;
  for (int w = 0; w < kCombThreads / 32; ++w) S += s_warp[w];
  const double pre = wpre + excl;
  const double nxt = wpre + incl;
  const double u = (double)a.u_draft[b * a.gamma + k];
  const double t = u * S;
  if (tid == 0) {
    s_chunk = -1;
    s_S = S;
    s_t = t;
  }
  __syncthreads();
  const bool last_nonempty = (c0 < c1) && (c1 == nchunk);
  if (c0 < c1 && pre <= t && (t < nxt || last_nonempty)) {
    double R = pre;
    int cf = -1, clast = -1;
    double Rlast = pre;
    for (int c = c0; c < c1; ++c) {
      const double w = (double)sm_s[c] * exp((double)sm_m[c] - Md);
      if (w > 0.0) {
        clast = c;
        Rlast = R;
      }
      if (t < R + w) {
        cf = c;
        break;
      }
      R += w;
    }
    if (cf < 0) {
      cf = clast;
      R = Rlast;
    }
    if (cf >= 0) {
      s_chunk = cf;
      s_base = R;
    }
  }
  __syncthreads();
  if (s_chunk < 0) {
    // every weight zero or non-finite: no valid distribution
    if (tid == 0) {
      int x = 0;
      for (int c = 0; c < nchunk; ++c)
        if (sm_m[c] == M) {
          x = c * kChunk;
          break;
        }
      atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
      a.x_out[b * a.gamma + k] = min(x, a.V - 1);
    }
    return;
  }
  if (warp == 0) {
    const int c = s_chunk;
    const int v = c * kChunk + lane;
    const bool valid = v < a.V;
    double e = 0.0;
    if (valid) {
      const float l = a.ld[((size_t)b * a.gamma + k) * a.V + v];
      const float z = __fmul_rn(l, a.inv_T);
      e = exp((double)z - Md);
    }
    const double base = s_base, Stot = s_S, tt = s_t;
    const double inc = warp_incl_scan_d(e);
    const double upper = base + inc, lower = upper - e;
    const unsigned cross = __ballot_sync(0xffffffffu, valid && e > 0.0 && tt < upper);
    int pick;
    if (cross) {
      pick = __ffs(cross) - 1;
    } else {
      const unsigned pos = __ballot_sync(0xffffffffu, valid && e > 0.0);
      pick = pos ? 31 - __clz(pos) : 0;
    }
    const double lo = __shfl_sync(0xffffffffu, lower, pick);
    const double hi = __shfl_sync(0xffffffffu, upper, pick);
    if (lane == 0) {
      const int x = min(c * kChunk + pick, a.V - 1);
      if ((tt - lo) < 1e-6 * Stot || (hi - tt) < 1e-6 * Stot) atomicOr(a.flags + b, DSPARK_FLAG_DRAFT_NEAR_TIE);
      if (!(Stot > 0.0) || !isfinite(Stot)) atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
      a.x_out[b * a.gamma + k] = x;
    }
  }
}

// ============================================================================ host side

size_t draft_workspace_bytes(int B, int gamma, int V, int r) {
  (void)gamma;
  (void)r;
  const size_t nchunk = (size_t)(V + kChunk - 1) / kChunk;
  return kWsHeader + align_up((size_t)B * nchunk * sizeof(ChunkStat), 256);
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, void* base, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  uint32_t es[3] = {1, 1, 1};
  CUresult rc = fn(m, dt, rank, base, dims, strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

template <typename K, typename... Args>
static cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename WT, int BG>
static cudaError_t launch_fma(const DraftArgs& a, int k, cudaStream_t st, bool pdl) {
  const int vec_ok = (a.V % (int)(16 / sizeof(WT)) == 0 && (uintptr_t)a.W2 % 16 == 0) ? 1 : 0;
  const size_t smem = (align_up((size_t)BG * a.r, 4) + (size_t)4 * BG * 256) * sizeof(float);
  auto kern = draft_main_fma<WT, BG>;
  static cudaError_t attr_rc = cudaSuccess;
  static size_t attr_smem = 0;
  if (smem > attr_smem) {
    attr_rc = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr_smem = smem;
  }
  if (attr_rc != cudaSuccess) return attr_rc;
  dim3 grid((a.V + 255) / 256, (a.B + BG - 1) / BG);
  return launch_ex(kern, grid, dim3(128), smem, st, pdl, a, k, vec_ok);
}

template <typename WT>
static cudaError_t launch_fma_bg(const DraftArgs& a, int k, cudaStream_t st, bool pdl) {
  if (a.B <= 1) return launch_fma<WT, 1>(a, k, st, pdl);
  if (a.B <= 2) return launch_fma<WT, 2>(a, k, st, pdl);
  if (a.B <= 4) return launch_fma<WT, 4>(a, k, st, pdl);
  return launch_fma<WT, 8>(a, k, st, pdl);
}

dspark_status launch_draft(const DraftCall& c) {
  const Options& opt = options();
  DraftArgs a{};
  a.U = c.U;
  a.W1 = c.W1;
  a.W2 = c.W2;
  a.x0 = c.x0;
  a.x_out = c.x_out;
  a.ld = c.ld_out;
  a.u_draft = c.u_draft;
  a.flags = c.flags;
  a.status = reinterpret_cast<uint32_t*>(c.ws);
  a.part = reinterpret_cast<ChunkStat*>(static_cast<uint8_t*>(c.ws) + kWsHeader);
  a.B = c.B;
  a.gamma = c.gamma;
  a.V = c.V;
  a.r = c.r;
  a.nchunk = (c.V + kChunk - 1) / kChunk;
  a.greedy = (c.T == 0.f) ? 1 : 0;
  a.inv_T = a.greedy ? 1.f : 1.f / c.T;
  const bool pdl = opt.draft_pdl != 0;

  const bool aligned16 = ((uintptr_t)c.U % 16 == 0) && ((uintptr_t)c.W1 % 16 == 0) &&
                         ((uintptr_t)c.W2 % 16 == 0) && ((uintptr_t)c.ld_out % 16 == 0);
  const bool tc_ok = c.w_dtype == DSPARK_BF16 && c.r % 64 == 0 && c.r <= 256 && c.V % 8 == 0 && aligned16;
  bool use_tc = tc_ok && c.B >= opt.draft_tc_min_b;
  if (opt.draft_force_path == 1) use_tc = false;
  if (opt.draft_force_path == 2) {
    if (!tc_ok) {
      set_error("tensor-core draft path forced but the shape or dtype does not allow it");
      return DSPARK_ENOTIMPL;
    }
    use_tc = true;
  }

  cudaError_t rc = cudaMemsetAsync(c.ws, 0, kWsHeader, c.stream);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaMemsetAsync: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }

  CUtensorMap mW2, mU, mLD;
  int n_bgroups = 1, cpg = 1, ntiles = 0, box_rows = 0;
  size_t tc_smem = 0;
  if (use_tc) {
    ntiles = (c.V + kTcN - 1) / kTcN;
    n_bgroups = (c.B + 127) / 128;
    const int sms = device_sm_count();
    cpg = std::max(1, sms / n_bgroups);
    cpg = std::min(cpg, ntiles);
    box_rows = std::min(128, (c.B + 7) / 8 * 8);
    {
      uint64_t dims[2] = {(uint64_t)c.V, (uint64_t)c.r};
      uint64_t strides[1] = {(uint64_t)c.V * 2};
      uint32_t box[2] = {64, (uint32_t)c.r};
      if (!make_map(&mW2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(c.W2), dims, strides, box)) {
        set_error("cuTensorMapEncodeTiled failed for W2");
        return DSPARK_ECUDA;
      }
    }
    {
      uint64_t dims[3] = {(uint64_t)c.V, (uint64_t)c.gamma, (uint64_t)c.B};
      uint64_t strides[2] = {(uint64_t)c.V * 4, (uint64_t)c.gamma * c.V * 4};
      uint32_t box[3] = {32, 1, (uint32_t)box_rows};
      if (!make_map(&mU, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(c.U), dims, strides, box) ||
          !make_map(&mLD, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, c.ld_out, dims, strides, box)) {
        set_error("cuTensorMapEncodeTiled failed for U / l_d");
        return DSPARK_ECUDA;
      }
    }
    tc_smem = tc_layout(c.r, box_rows).total + 1024;
    static size_t attr_smem = 0;
    if (tc_smem > attr_smem) {
      rc = cudaFuncSetAttribute(draft_main_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem);
      if (rc != cudaSuccess) {
        set_error(std::string("cudaFuncSetAttribute(draft_main_tc): ") + cudaGetErrorString(rc));
        return DSPARK_ECUDA;
      }
      attr_smem = tc_smem;
    }
  }

  const size_t comb_smem = a.greedy ? 0 : (size_t)2 * a.nchunk * sizeof(float);
  {
    static size_t attr_smem = 0;
    if (comb_smem > 48 * 1024 && comb_smem > attr_smem) {
      rc = cudaFuncSetAttribute(draft_combine, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)comb_smem);
      if (rc != cudaSuccess) {
        set_error(std::string("cudaFuncSetAttribute(draft_combine): ") + cudaGetErrorString(rc));
        return DSPARK_ECUDA;
      }
      attr_smem = comb_smem;
    }
  }

  for (int k = 0; k < c.gamma; ++k) {
    // The first main pass waits for everything before the call in full: its TMA producer reads
    // U and W2 without a grid-dependency wait, which is only safe behind this call's own kernels.
    const bool pdl_k = pdl && k > 0;
    if (use_tc) {
      rc = launch_ex(draft_main_tc, dim3(cpg * n_bgroups), dim3(kTcThreads), tc_smem, c.stream, pdl_k, mW2, mU, mLD,
                     a, k, ntiles, n_bgroups, cpg, box_rows);
    } else if (c.w_dtype == DSPARK_BF16) {
      rc = launch_fma_bg<__nv_bfloat16>(a, k, c.stream, pdl_k);
    } else {
      rc = launch_fma_bg<float>(a, k, c.stream, pdl_k);
    }
    if (rc != cudaSuccess) {
      set_error(std::string("draft main pass launch: ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
    rc = launch_ex(draft_combine, dim3(c.B), dim3(kCombThreads), comb_smem, c.stream, pdl, a, k);
    if (rc != cudaSuccess) {
      set_error(std::string("draft combine launch: ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  }
  return DSPARK_OK;
}

}  // namespace dspark
