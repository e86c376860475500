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
//   combine    -- per request: global max and normaliser from the per-partition statistics
//                 (fp64 sums), the partition that crosses u * S, a rescan of that partition's
//                 stored logits for x_k and the near-tie flag.
// The main pass of step k+1 prefetches its W2 / U tiles before waiting on step k's combine.

#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
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
  ChunkStat* cpart;    // [np][B]: per (main-pass partition, request) statistics
  __nv_bfloat16* gbuf; // [B][r]: W1 rows of the tokens just drafted (next step's B operand), or null
  uint32_t* status;
  size_t sk, sb;         // element strides of the U / l_d row of position k and request b
  int rm;                // 1: request-major U / l_d ([B][gamma][V]; tensor maps {V, gamma, B})
  uint32_t spin_limit;   // polls before a bounded wait gives up
  int barrier_extra;     // test-only: arrivals the first grid barrier expects beyond the grid
  const void* Wh;        // recurrent head: [r][r] state matrix, or null (Markov head)
  float* hstate;         // recurrent head: [B][r] fp32 state h_k of the step being drafted
  float* h_out;          // recurrent head: [B][gamma][r] copy of every state, or null
  int B, gamma, V, r, nchunk;
  float inv_T;
  int greedy;
  int np;              // partitions of the vocabulary: partition p covers tiles
  int ntiles;          //   [p*ntiles/np, (p+1)*ntiles/np) of tile_chunks chunks each
  int tile_chunks;
};

// Fold statistics of a disjoint column range into `acc`: (max, sum of exp) pairs, or greedy top-2.
__device__ __forceinline__ void stat_fold(ChunkStat& acc, const ChunkStat& o, int greedy) {
  if (greedy) {
    const Top2 r = top2_merge(Top2{acc.m, acc.idx, acc.m2}, Top2{o.m, o.idx, o.m2});
    acc.m = r.best;
    acc.idx = r.idx;
    acc.m2 = r.second;
  } else {
    const float M = fmaxf(acc.m, o.m);
    if (M == -INFINITY) {
      acc.s = 0.f;
    } else {
      acc.s = acc.s * exp2f(__fmul_rn(__fsub_rn(acc.m, M), kLog2e)) + o.s * exp2f(__fmul_rn(__fsub_rn(o.m, M), kLog2e));
    }
    acc.m = M;
  }
}

__device__ __forceinline__ ChunkStat stat_empty() { return ChunkStat{-INFINITY, 0.f, -1, -INFINITY}; }

// exp(z - m) as 2^((z - m) log2 e); z and m are already-rounded fp32 values
__device__ __forceinline__ float ex_shift(float z, float m) { return exp2f(__fmul_rn(__fsub_rn(z, m), kLog2e)); }

__device__ __forceinline__ int prev_token(const DraftArgs& a, int b, int k, bool report) {
  int prev = (k == 0) ? a.x0[b] : __ldcg(a.x_out + b * a.gamma + k - 1);  // may be this launch's
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

// Grid: x = 256-column tile (one partition of the combine's first level), y = group of BG
// requests.  128 threads: the rank dimension r is split over the 4 warps, each lane owns 8
// consecutive columns; the partial sums meet in shared memory, then every thread finishes 2
// columns for each request of the group.
template <typename WT, int BG>
__global__ void __launch_bounds__(128) draft_main_fma(DraftArgs a, int k, int vec_ok) {
  extern __shared__ __align__(16) float fsm[];
  __shared__ ChunkStat s_stat[8][BG];
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
    if (bb < nb)
      g = a.hstate ? a.hstate[(size_t)(b0 + bb) * r + kk]  // recurrent head: the state h_k
                   : wload<WT>(a.W1, (size_t)prev_token(a, b0 + bb, k, kk == 0) * r + kk);
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
  const int lchunk = tid >> 4;  // chunk of this CTA, 0..7
  const int chunk = v0 / kChunk + lchunk;
  for (int bb = 0; bb < nb; ++bb) {
    const int b = b0 + bb;
    float bias0 = 0.f, bias1 = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      bias0 += red[(w * BG + bb) * 256 + c];
      bias1 += red[(w * BG + bb) * 256 + c + 1];
    }
    const size_t row = (size_t)k * a.sk + (size_t)b * a.sb;
    float l0 = 0.f, l1 = 0.f;
    if (val0) {
      l0 = a.U[row + v] + bias0;
      a.ld[row + v] = l0;
    }
    if (val1) {
      l1 = a.U[row + v + 1] + bias1;
      a.ld[row + v + 1] = l1;
    }
    if ((val0 && (isnan(l0) || l0 == INFINITY)) || (val1 && (isnan(l1) || l1 == INFINITY)))
      atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
    const ChunkStat st = chunk_stat_pair(l0, l1, val0, val1, v, a.inv_T, a.greedy);
    if ((tid & 15) == 0) s_stat[lchunk][bb] = chunk < a.nchunk ? st : stat_empty();
  }
  __syncthreads();
  if (tid < nb) {  // fold the CTA's 8 chunks into its partition record
    ChunkStat acc = s_stat[0][tid];
    for (int q = 1; q < 8; ++q) stat_fold(acc, s_stat[q][tid], a.greedy);
    a.cpart[(size_t)blockIdx.x * a.B + b0 + tid] = acc;
  }
}

// ============================================================================ recurrent head state
//
// [P1 §DSpark 架构设计：半自回归生成与马尔可夫修正: the optional RNN head keeps a hidden state over
//  the whole drafted prefix; P3 §Semi-Autoregressive Generation: B_k(x_<k, v) from a recurrent
//  state inside the block]  The pages give no form; the state here has the Markov head's rank r:
//      h_k = tanh(W1[x_{k-1}] + h_{k-1} W_h),  h_{-1} = 0,  x_{-1} = x0,   bias_k = h_k W2,
// in fp32 (the contraction over W_h sums i = 0..r-1 in order with fused multiply-adds).  One CTA
// per request, one thread per state element; the main pass then reads h_k where the Markov head
// reads W1[x_{k-1}].  The state stays fp32 on the CUDA-core pass (the tensor-core pass would
// have to round it to bf16 for its operand).

template <typename WT>
__global__ void __launch_bounds__(256) rnn_state_kernel(DraftArgs a, int k) {
  extern __shared__ float hp[];  // [r]: h_{k-1}
  const int b = blockIdx.x, r = a.r;
  float* h = a.hstate + (size_t)b * r;
  for (int j = threadIdx.x; j < r; j += blockDim.x) hp[j] = k == 0 ? 0.f : h[j];
  __syncthreads();  // every read of this request's state precedes the writes below
  const int prev = prev_token(a, b, k, threadIdx.x == 0);
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    float pre = wload<WT>(a.W1, (size_t)prev * r + j);
    for (int i = 0; i < r; ++i) pre = fmaf(hp[i], wload<WT>(a.Wh, (size_t)i * r + j), pre);
    const float hj = tanhf(pre);
    h[j] = hj;
    if (a.h_out) a.h_out[((size_t)b * a.gamma + k) * r + j] = hj;
  }
}

// ============================================================================ tcgen05 main pass
//
// One CTA per SM over a contiguous run of 128-column tiles of the vocabulary (one partition of
// the combine's first level), for one group of NB requests (NB = 32 or 64; larger batches use
// several groups).  The MMA computes the bias tile transposed, D[v][b] = sum_k W2[k][v] B[b][k]:
// M = 128 vocabulary columns on the TMEM lanes and N = NB requests on the TMEM columns, so no
// MMA row is padding.
//   warp 0      TMA producer: the W2 tile [r x 128] bf16 as two 64-column boxes (MN-major A
//               operand, 128-byte swizzle) in a 2-stage ring.
//   warp 1      MMA issuer: r/16 tcgen05.mma kind::f16 (M = 128, N = NB, K = 16) per tile into
//               one of two TMEM accumulators of NB fp32 columns.
//   warp 2      TMEM allocation owner.
//   warp 3      U and l_d: one TMA box per tile brings U [NB requests x 128 columns] (32 KB at
//               NB = 64) into a 2-stage buffer; when the epilogue has written l = U + bias in
//               place, one TMA store writes the tile of l_d and the stage is refilled two tiles
//               ahead (copies this size keep the copy engine near full HBM bandwidth; 4 KB ones
//               were measured to stream at under half).
//   warps 4..   epilogue, NB/8 warps: warp w owns TMEM lane quadrant w%4 (32 vocabulary columns)
//               for the 32 requests of its column group: it adds the bias to its [32 x 32] block
//               of the U stage (lane = column), then each lane reads its own request's row
//               (rotated 16-byte chunks, free of bank conflicts) and reduces the chunk statistics
//               sequentially.  The statistics are also folded into one record per (CTA, request)
//               for the combine's first level.
// The B operand (the gathered W1 rows, K-major, 128-byte swizzle) is built once per step.

constexpr int kTcTile = 128;
constexpr int kTcThreads = 384;
constexpr int kTcStages = 2;

struct TcLayout {
  uint32_t g, w2, u, bars, misc, total;
  uint32_t w2_stage_bytes;
};

__host__ __device__ inline TcLayout tc_layout(int r, int nb) {
  TcLayout L;
  L.g = 0;
  L.w2_stage_bytes = (uint32_t)r * 256u;  // two 64-column atoms of r rows x 128 B
  L.w2 = ((uint32_t)nb * (uint32_t)r * 2u + 1023u) & ~1023u;
  L.u = L.w2 + kTcStages * L.w2_stage_bytes;
  L.bars = L.u + 2u * (uint32_t)nb * kTcTile * 4u;  // two [nb requests x 128 columns] fp32 stages
  L.misc = L.bars + 8u * (2 * kTcStages + 2 + 2 + 1 + 2 + 2 + 2 + 1);
  L.total = L.misc + 16u;
  return L;
}

struct TcSync {
  volatile int* abort;
  uint32_t* status;
  uint32_t limit;  // polls before a wait gives up
};

// Bounded mbarrier wait shared by all roles; after any timeout every later wait returns at once.
__device__ __forceinline__ bool tc_wait(const TcSync& s, uint64_t* bar, uint32_t parity) {
  if (*s.abort) return false;
  for (uint32_t i = 0; i < s.limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *s.abort) return false;
  }
  *s.abort = 1;
  atomicOr(s.status, (uint32_t)DSPARK_ETIMEOUT);
  return false;
}

// A group of nth threads (a multiple of 32, ranks tid = 0..nth-1) that synchronises with
// __syncthreads (bar < 0) or with named barrier `bar`.
struct Grp {
  int tid, nth, bar;
  __device__ __forceinline__ void sync() const {
    if (bar < 0) __syncthreads();
    else named_bar(bar, nth);
  }
};

// Inclusive fp64 scan over the group in rank order; `total` gets the group's sum.  sh: >= 33 doubles.
__device__ __forceinline__ double grp_incl_scan_d(double v, double* sh, const Grp& g, double& total) {
  const int lane = g.tid & 31, w = g.tid >> 5, nw = g.nth >> 5;
  v = warp_incl_scan_d(v);
  if (lane == 31) sh[w] = v;
  g.sync();
  if (w == 0) {
    double x = lane < nw ? sh[lane] : 0.0;
    x = warp_incl_scan_d(x);
    if (lane < nw) sh[lane] = x;
  }
  g.sync();
  const double pre = w > 0 ? sh[w - 1] : 0.0;
  total = sh[nw - 1];
  g.sync();
  return v + pre;
}

__device__ __forceinline__ float grp_max_f(float v, float* sh, const Grp& g) {
  const int lane = g.tid & 31, w = g.tid >> 5, nw = g.nth >> 5;
  v = warp_max(v);
  if (lane == 0) sh[w] = v;
  g.sync();
  float r = sh[0];
  for (int i = 1; i < nw; ++i) r = fmaxf(r, sh[i]);
  g.sync();
  return r;
}

// Grid-wide barrier of the multi-step launch (cooperative, so every CTA is resident): one thread
// per CTA after a CTA-level barrier adds 1 to a monotonic counter with a release reduction (no
// returned value, so the arrivals do not queue on each other) and waits, with acquire loads, for
// it to reach nblocks times the barrier's number.  Bounded: gives up with the timeout status and
// the abort flag.
__device__ __forceinline__ bool grid_sync(uint32_t* count, uint32_t nblocks, uint32_t& epoch, const TcSync& sy,
                                          uint32_t extra = 0) {
  if (*sy.abort) return false;
  const uint32_t target = ++epoch * nblocks + extra;
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(count) : "memory");
  for (uint32_t i = 0; i < sy.limit; ++i) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(count) : "memory");
    if ((int32_t)(v - target) >= 0) return true;
    if ((i & 1023u) == 1023u && *sy.abort) return false;
  }
  *sy.abort = 1;
  atomicOr(sy.status, (uint32_t)DSPARK_ETIMEOUT);
  return false;
}

__device__ void combine_group(const DraftArgs& a, int k, int b, const Grp& g, double* sh);
__device__ void combine_warp(const DraftArgs& a, int k, int b, uint32_t* gready);

// Steps k0 .. k1-1 of the draft.  With fused = 0 the launch is one step and a separate combine
// kernel samples its tokens; with fused = 1 (a cooperative launch, all CTAs resident) every step
// ends with a grid barrier, the combine of that step inside the kernel (the epilogue warps take one
// request each) and a second grid barrier, after which the next step gathers its W1 rows.  The
// W2 and U streams run on across steps (tile counter gi = step * nt + tile), so the next step's
// first tiles are already loaded when its gather finishes.
template <int NB>
__global__ void __launch_bounds__(kTcThreads, 1)
    draft_main_tc(const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmU,
                  const __grid_constant__ CUtensorMap tmLd, const __grid_constant__ CUtensorMap tmG, DraftArgs a,
                  int k0, int k1, int n_bgroups, int ctas_per_group, int fused) {
  constexpr int EPI_WARPS = NB / 8;  // 4 per 32-request column group
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const TcLayout L = tc_layout(a.r, NB);
  uint8_t* sG = sm + L.g;
  uint8_t* sW = sm + L.w2;
  float* sU = reinterpret_cast<float*>(sm + L.u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* w_full = bars;
  uint64_t* w_empty = w_full + kTcStages;
  uint64_t* t_full = w_empty + kTcStages;
  uint64_t* t_empty = t_full + 2;
  uint64_t* mma_done = t_empty + 2;
  uint64_t* u_full = mma_done + 1;  // [2] U stage landed
  uint64_t* u_empty = u_full + 2;   // [2] every epilogue warp is done reading the stage
  uint64_t* c_done = u_empty + 2;   // [2] every epilogue warp has written l = U + bias in place
  uint64_t* g_full = c_done + 2;    // the B operand arrived by TMA from gbuf
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.misc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L.misc + 4);
  const TcSync sy{s_abort, a.status, a.spin_limit};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x % n_bgroups;
  const int jc = blockIdx.x / n_bgroups;
  // This CTA's columns are half-tiles [h_beg, h_end) of 64 columns (a.ntiles of them in V), so
  // the CTAs' shares differ by at most 64 columns; it runs them as 128-column tiles starting at
  // h_beg, the last one half when the count is odd.  A half tile still computes, loads and stores
  // 128 columns (its second half is the next CTA's first, and the values written are the same
  // bits: the same inputs through the same MMA), but only its own 64 enter the statistics.
  const int h_beg = (int)((long long)jc * a.ntiles / ctas_per_group);
  const int h_end = (int)((long long)(jc + 1) * a.ntiles / ctas_per_group);
  const int nt = (h_end - h_beg + 1) / 2;
  const bool last_half = ((h_end - h_beg) & 1) != 0;
  auto tile_col = [&](int i) { return (h_beg + 2 * i) * 64; };  // first column of tile i
  const int b0 = g * NB;
  const int ksteps = a.r / 16;
  const int total = (k1 - k0) * nt;  // tiles of this CTA over the launch

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(&w_full[i], 1);
      mbar_init(&w_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&t_full[i], 1);
      mbar_init(&t_empty[i], EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&u_full[i], 1);
      mbar_init(&u_empty[i], EPI_WARPS);
      mbar_init(&c_done[i], EPI_WARPS);
    }
    mbar_init(g_full, 1);
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tmW2);
    prefetch_tmap(&tmU);
    prefetch_tmap(&tmLd);
    if (a.gbuf) prefetch_tmap(&tmG);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 2 * NB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_trigger();

  // epilogue geometry (warps 4 .. 4+EPI_WARPS-1)
  const bool epi = warp >= 4 && warp < 4 + EPI_WARPS;
  const int q = warp & 3, h = (warp - 4) >> 2;
  const int bb = b0 + h * 32;
  constexpr uint32_t kUStage = (uint32_t)NB * kTcTile;  // floats of one U stage: [NB requests][128 columns]
  // U (an input of the call) for the first two tiles is requested before waiting for the previous
  // kernel: one 128-column x NB-request box per tile.  L2 policies: U and l_d, streamed once per
  // step, are evict-first; W2, read at every step, is evict-last on half of its lines (the
  // setting measured fastest at B = 64, gamma = 16: 562 against 595 us without policies; W2
  // evict-last on every line, 587 us).
  auto load_u = [&](int gi) {
    const int j = gi & 1, ku = k0 + gi / nt, iu = gi % nt;
    mbar_arrive_expect_tx(&u_full[j], kUStage * 4u);
    tma_load_3d_hint(sU + j * kUStage, &tmU, tile_col(iu), a.rm ? ku : b0, a.rm ? b0 : ku, &u_full[j],
                     l2_policy_evict_first());
  };
  if (warp == 3 && lane == 0)
    for (int gi = 0; gi < 2 && gi < total; ++gi) load_u(gi);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // W2 is an input of the call: the ring fills before the previous kernel has finished, and
    // across steps (the same tiles every step).
    if (lane == 0) {
      int issued = 0;
      for (int gi = 0; gi < total; ++gi) {
        // a half tile loads its whole W2 tile too: its upper 64 columns are stored as well
        const int v0 = tile_col(gi % nt);
        const int s = gi % kTcStages;
        if (!tc_wait(sy, &w_empty[s], ((gi / kTcStages) & 1) ^ 1)) break;
        uint8_t* st = sW + s * L.w2_stage_bytes;
        mbar_arrive_expect_tx(&w_full[s], L.w2_stage_bytes);
        const uint64_t pol = l2_policy_evict_last_half();
        tma_load_2d_hint(st, &tmW2, v0, 0, &w_full[s], pol);
        tma_load_2d_hint(st + L.w2_stage_bytes / 2, &tmW2, v0 + 64, 0, &w_full[s], pol);
        issued = gi + 1;
      }
      if (*s_abort) {
        // give the copies already issued a bounded chance to land before the CTA exits
        for (int i = max(0, issued - kTcStages); i < issued; ++i)
          for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(&w_full[i % kTcStages], (i / kTcStages) & 1); ++t) {
          }
      }
    }
  } else {
    // All other warps walk the steps together: every named barrier below is reached by all of
    // them on every step, also after a timeout (the waits then return at once).
    pdl_wait();
    uint32_t epoch = 0;
    uint32_t* gcount = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.status) + 64);
    uint32_t* gready = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(a.status) + 128);
    bool bad = false;
    int last_load[2] = {total > 0 ? 0 : -1, total > 1 ? 1 : -1};  // (warp 3) last tile loaded into each U stage
    int g_issued = 0;  // (warp 1) TMA loads of the B operand issued
    for (int k = k0; k < k1; ++k) {
      const int gbase = (k - k0) * nt;
      // ---------------------------------------------------------------- B operand = W1[x_{k-1}] rows
      // Step 0 gathers the rows of x0; later steps load the rows the previous combine copied to
      // gbuf, with r/64 TMA boxes of [NB rows x 64 columns] (the same 128-byte swizzled K-major
      // layout as the gather writes).
      const bool tma_g = a.gbuf != nullptr && k > 0;
      if (!tma_g) {
        const int cpr = a.r / 8;  // 16-byte chunks per row
        const __nv_bfloat16* W1 = static_cast<const __nv_bfloat16*>(a.W1);
        for (int i = threadIdx.x - 32; i < NB * cpr; i += kTcThreads - 32) {
          const int row = i / cpr, c = i - row * cpr;
          const int b = b0 + row;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (b < a.B)
            val = __ldg(reinterpret_cast<const uint4*>(W1 + (size_t)prev_token(a, b, k, c == 0) * a.r + c * 8));
          const int kb = c >> 3, cc = c & 7;
          *reinterpret_cast<uint4*>(sG + kb * (NB * 128) + row * 128 + ((cc ^ (row & 7)) << 4)) = val;
        }
        fence_proxy_async_smem();
      } else if (warp == 1 && lane == 0 && !*s_abort) {  // after a timeout nothing waits for it
        fence_proxy_async_smem();  // earlier generic accesses to the G region come first
        mbar_arrive_expect_tx(g_full, (uint32_t)NB * a.r * 2u);
        for (int kb = 0; kb < a.r / 64; ++kb) tma_load_2d(sG + kb * (NB * 128), &tmG, kb * 64, b0, g_full);
        ++g_issued;
      }
      named_bar(1, kTcThreads - 32);
      if (warp == 3) {
        // ---------------------------------------------------------------- U refills and l_d stores
        // l_d = U + bias is written in place in the U stage by the epilogue; one TMA store per tile
        // writes it out, and the stage is refilled with the U tile two ahead (possibly of the next
        // step) once the store has read it and every epilogue warp is done with it.
        if (lane == 0) {
          for (int i = 0; i < nt; ++i) {
            const int gi = gbase + i, j = gi & 1;
            if (!tc_wait(sy, &c_done[j], (gi >> 1) & 1)) break;
            tma_store_3d_hint(&tmLd, sU + j * kUStage, tile_col(i), a.rm ? k : b0, a.rm ? b0 : k,
                              l2_policy_evict_first());
            bulk_commit();
            if (gi + 2 < total) {
              if (!tc_wait(sy, &u_empty[j], (gi >> 1) & 1)) break;
              bulk_wait_read0();
              load_u(gi + 2);
              last_load[j] = gi + 2;
            }
          }
          bulk_wait0();     // this step's l_d is written before anyone samples from it
          __threadfence();
        }
        __syncwarp();
      } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
          const uint32_t idesc = (1u << 4)                       // D fp32
                                 | (1u << 7) | (1u << 10)        // A, B bf16
                                 | (1u << 15)                    // A MN-major (W2 is [r][V])
                                 | ((uint32_t)(NB >> 3) << 17)   // N
                                 | ((uint32_t)(128 >> 4) << 24);  // M
          const uint32_t g_addr = smem_u32(sG), w_addr = smem_u32(sW);
          // the n-th TMA load of the B operand in this launch completes phase n of g_full
          const bool g_ok = !tma_g || tc_wait(sy, g_full, (uint32_t)(k - max(k0, 1)) & 1u);
          for (int i = 0; g_ok && i < nt; ++i) {
            const int gi = gbase + i, acc = gi & 1, s = gi % kTcStages;
            if (!tc_wait(sy, &t_empty[acc], ((gi >> 1) & 1) ^ 1)) break;
            if (!tc_wait(sy, &w_full[s], (gi / kTcStages) & 1)) break;
            tc_fence_after();
            const uint32_t wst = w_addr + s * L.w2_stage_bytes;
            for (int kk = 0; kk < ksteps; ++kk) {
              const uint64_t ad = smem_desc(wst + kk * 2048u, L.w2_stage_bytes / 2, 1024u, 2u);
              const uint64_t bd = smem_desc(g_addr + (kk >> 2) * (NB * 128u) + (kk & 3) * 32u, 16u, 1024u, 2u);
              tc_mma_f16(tmem_base + acc * NB, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(&w_empty[s]);
            tc_commit(&t_full[acc]);
          }
        }
        __syncwarp();
      } else if (epi) {
        // ---------------------------------------------------------------- epilogue
        const float inv_T = a.inv_T;
        const int b = bb + lane;  // this lane's request in the row phase
        const bool bok = b < a.B;
        ChunkStat run = stat_empty();
        for (int i = 0; i < nt; ++i) {
          const int gi = gbase + i, j = gi & 1, acc = gi & 1;
          const int v0w = tile_col(i) + q * 32;  // this warp's 32 columns
          const bool own = !(last_half && i == nt - 1 && q >= 2);  // columns of this CTA
          const bool ok_u = tc_wait(sy, &u_full[j], (gi >> 1) & 1);
          const bool ok_t = __all_sync(0xffffffffu, tc_wait(sy, &t_full[acc], (gi >> 1) & 1) && ok_u);
          float x[32];
          if (ok_t) {
            tc_fence_after();
            tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * NB + h * 32, x);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&t_empty[acc]);
          // this warp's [32 requests x 32 columns] block of the stage (row stride 128 columns)
          float* ub = sU + j * kUStage + (h * 32) * kTcTile + q * 32;
          if (ok_t) {
            // column phase: lane = column, row jj = request: l = U + bias in place
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) ub[jj * kTcTile + lane] += x[jj];
            fence_proxy_async_smem();  // the TMA store reads these values
            __syncwarp();
            if (lane == 0) mbar_arrive(&c_done[j]);
            // row phase: lane = request; rotated 16-byte chunks keep the eight lanes of each
            // shared-memory phase on distinct banks
            float lv[32];
#pragma unroll
            for (int s4 = 0; s4 < 8; ++s4) {
              const int c = (lane + s4) & 7;
              const float4 f = *reinterpret_cast<const float4*>(ub + lane * kTcTile + c * 4);
              lv[4 * s4 + 0] = f.x;
              lv[4 * s4 + 1] = f.y;
              lv[4 * s4 + 2] = f.z;
              lv[4 * s4 + 3] = f.w;
            }
            const int nval = own ? min(32, a.V - v0w) : 0;  // valid columns of this chunk (multiple of 8)
            ChunkStat st;
            if (a.greedy) {
              Top2 t{-INFINITY, -1, -INFINITY};
#pragma unroll
              for (int s4 = 0; s4 < 8; ++s4) {
                const int c = (lane + s4) & 7;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int col = c * 4 + e;
                  const float l = lv[4 * s4 + e];
                  if (col < nval) {
                    bad |= isnan(l) || l == INFINITY;
                    const Top2 o{l, v0w + col, -INFINITY};
                    t = top2_merge(t, o);
                  }
                }
              }
              st = ChunkStat{t.best, 0.f, t.idx, t.second};
            } else {
              float mx = -INFINITY;
#pragma unroll
              for (int s4 = 0; s4 < 8; ++s4) {
                const int c = (lane + s4) & 7;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  lv[4 * s4 + e] = (c * 4 + e < nval) ? __fmul_rn(lv[4 * s4 + e], inv_T) : -INFINITY;  // z
                  mx = fmaxf(mx, lv[4 * s4 + e]);
                }
              }
              float sm = 0.f;
#pragma unroll
              for (int e = 0; e < 32; ++e) sm += (lv[e] == -INFINITY) ? 0.f : ex_shift(lv[e], mx);
              bad |= isnan(sm) || mx == INFINITY;
              st = ChunkStat{mx, sm, 0, 0.f};
            }
            if (own && v0w < a.V) stat_fold(run, st, a.greedy);
          }
          __syncwarp();  // every lane is done with this stage
          if (lane == 0) mbar_arrive(&u_empty[j]);
        }
        // partition record: fold the four lane quadrants (through shared memory: the G region,
        // free once every MMA of the step has completed, which the last accumulator wait
        // guarantees)
        ChunkStat* comb = reinterpret_cast<ChunkStat*>(sG);
        comb[q * NB + h * 32 + lane] = run;
        named_bar(2, EPI_WARPS * 32);
        if (q == 0 && bok) {
          ChunkStat r = comb[h * 32 + lane];
          for (int qq = 1; qq < 4; ++qq) stat_fold(r, comb[qq * NB + h * 32 + lane], a.greedy);
          a.cpart[(size_t)jc * a.B + b] = r;
        }
        fence_proxy_async_smem();      // the next B operand arrives in the G region by TMA
        named_bar(2, EPI_WARPS * 32);  // the G region is read before anyone reuses it
      }
      if (fused) {
        // ---------------------------------------------------------------- sample this step
        // every CTA's partition records and l_d stores of the step are in place
        named_bar(3, kTcThreads - 32);
        if (warp == 1 && lane == 0) grid_sync(gcount, gridDim.x, epoch, sy, (uint32_t)a.barrier_extra);
        named_bar(3, kTcThreads - 32);
        // one warp per request, the requests spread over the grid (request blockIdx.x + m*gridDim.x
        // goes to warp 1 + m % 11 of this CTA): no block barrier inside a combine
        for (int m = 0;; ++m) {
          const int rq = (int)blockIdx.x + m * (int)gridDim.x;
          if (rq >= a.B) break;
          if (warp == 1 + m % (kTcThreads / 32 - 1)) combine_warp(a, k, rq, gready);
        }
        // the next step's B operand needs the W1 rows of all B tokens just drafted: each combine
        // counts its row in; the MMA warp waits for the step's B rows before it loads them
        if (k + 1 < k1 && a.gbuf) {
          if (warp == 1 && lane == 0) {
            const uint32_t target = (uint32_t)(k - k0 + 1) * (uint32_t)a.B;
            bool okc = !*s_abort;
            for (uint32_t i = 0; okc; ++i) {
              uint32_t v;
              asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(gready) : "memory");
              if ((int32_t)(v - target) >= 0) break;
              if (i >= a.spin_limit || ((i & 1023u) == 1023u && *s_abort)) {
                if (!*s_abort) {
                  *s_abort = 1;
                  atomicOr(a.status, (uint32_t)DSPARK_ETIMEOUT);
                }
                okc = false;
              }
            }
            // the rows were written with generic stores; the B operand is read by TMA
            asm volatile("fence.proxy.async.global;" ::: "memory");
          }
          named_bar(3, kTcThreads - 32);
        }
      }
    }
    if (epi) {
      const int b = bb + lane;
      if (bad && b < a.B) atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
    }
    if (warp == 3 && lane == 0 && *s_abort) {
      // let U copies still in flight land before the CTA exits
      for (int j = 0; j < 2; ++j)
        if (last_load[j] >= 0)
          for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(&u_full[j], (last_load[j] >> 1) & 1); ++t) {
          }
    }
    if (warp == 1 && lane == 0 && *s_abort && g_issued > 0) {
      // a B-operand copy issued before the timeout that no wait saw land: let it land
      for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(g_full, (uint32_t)(g_issued - 1) & 1u); ++t) {
      }
    }
    if (warp == 1 && lane == 0) tc_commit(mma_done);
  }
  __syncthreads();
  if (warp == 2) {
    // every MMA issued has to finish before the columns are released
    for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(mma_done, 0); ++t) {
    }
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * NB);
  }
  if (threadIdx.x == 0 && *s_abort && a.flags)
    for (int i = 0; i < min(NB, a.B - b0); ++i) atomicOr(a.flags + b0 + i, DSPARK_FLAG_DEVICE_TIMEOUT);
}

// ============================================================================ combine + sample
//
// One warp per request, two short levels, all weights exp(z - M) relative to the row maximum M:
//   1  the np partition records -> M, S and the partition holding u*S (fp64 warp scan over
//      contiguous ranges of records, exact partition of [0, S));
//   2  that partition's stored logits (about 1000 columns, each lane a contiguous run) -> the
//      token (and the near-tie flag).  The main passes keep no finer records: one more
//      dependent level cost more than the rescan.
// Greedy: the partition records already carry the argmax (lowest index) and the runner-up.

__device__ __forceinline__ ChunkStat ld_stat_cg(const ChunkStat* p) {
  const float4 v = __ldcg(reinterpret_cast<const float4*>(p));
  return ChunkStat{v.x, v.y, __float_as_int(v.z), v.w};
}

// Combine of one request by a whole group of threads (one element per thread per level, scans
// in fp64): partitions -> M, S and the partition holding u*S; that partition's stored logits ->
// the token x_k (and the near-tie flag).  Weights are exp(z - M) through exp2, as in the main
// passes.  Records and logits are read through L2 (ld.global.cg): in the multi-step launch other
// CTAs wrote them during this kernel.  The group then copies W1[x_k] into row b of `gbuf`
// (the next step's B operand) when gbuf is given.  sh: >= 72 doubles of shared memory.
__device__ void combine_group(const DraftArgs& a, int k, int b, const Grp& g, double* sh) {
  const size_t B = (size_t)a.B;
  const int np = a.np, nth = g.nth, tid = g.tid;
  double* shs = sh;                                   // scan scratch (33)
  float* shf = reinterpret_cast<float*>(sh + 34);     // max scratch (32 floats = 16 doubles)
  int* shi = reinterpret_cast<int*>(sh + 52);         // [0] pick, [1] token, [2] flags
  double* shd = sh + 56;                              // [0] lo of the pick, [1] hi
  // requested before the first dependent load; greedy drafting takes no uniforms (u_draft may be null)
  const float u = a.greedy ? 0.f : __ldg(a.u_draft + b * a.gamma + k);
  if (tid == 0) shi[0] = -1;

  if (a.greedy) {
    Top2 t{-INFINITY, -1, -INFINITY};
    for (int p = tid; p < np; p += nth) {
      const ChunkStat s = ld_stat_cg(a.cpart + p * B + b);
      t = top2_merge(t, Top2{s.m, s.idx, s.m2});
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t = top2_merge(t, top2_shfl_xor(t, o));
    Top2* sht = reinterpret_cast<Top2*>(sh);
    if ((tid & 31) == 0) sht[tid >> 5] = t;
    g.sync();
    if (tid == 0) {
      Top2 r = sht[0];
      for (int i = 1; i < nth / 32; ++i) r = top2_merge(r, sht[i]);
      int x = r.idx;
      uint32_t fl = 0;
      if (x < 0 || x >= a.V) {
        fl |= DSPARK_FLAG_NONFINITE;
        x = min(max(x, 0), a.V - 1);
      }
      if (r.best - r.second <= 1e-6f * fmaxf(1.f, fabsf(r.best))) fl |= DSPARK_FLAG_DRAFT_NEAR_TIE;
      if (fl) atomicOr(a.flags + b, fl);
      a.x_out[b * a.gamma + k] = x;
      shi[1] = x;
    }
    g.sync();
  } else {
    // ---- level 1: each thread a contiguous run of partition records
    const int e1 = (np + nth - 1) / nth;
    const int i0 = min(np, tid * e1), i1 = min(np, i0 + e1);
    float ml = -INFINITY;
    for (int i = i0; i < i1; ++i) ml = fmaxf(ml, ld_stat_cg(a.cpart + (size_t)i * B + b).m);
    const float M = grp_max_f(ml, shf, g);
    auto w1 = [&](int i) -> double {
      const ChunkStat s = ld_stat_cg(a.cpart + (size_t)i * B + b);
      return s.m == -INFINITY ? 0.0 : (double)s.s * (double)ex_shift(s.m, M);
    };
    double own = 0.0;
    for (int i = i0; i < i1; ++i) own += w1(i);
    double S = 0.0;
    const double incl = grp_incl_scan_d(own, shs, g, S);
    const double t = (double)u * S;
    {
      const double excl = incl - own;
      if (i0 < i1 && excl <= t && (t < incl || i1 == np)) {
        double R = excl;
        int pick = -1, last = -1;
        double plo = 0.0, lastlo = 0.0;
        for (int i = i0; i < i1; ++i) {
          const double w = w1(i);
          if (w > 0.0) {
            last = i;
            lastlo = R;
            if (t < R + w) {
              pick = i;
              plo = R;
              break;
            }
          }
          R += w;
        }
        if (pick < 0) {
          pick = last;
          plo = lastlo;
        }
        if (pick >= 0) {
          shi[0] = pick;
          shd[0] = plo;
        }
      }
    }
    g.sync();
    const int p = shi[0];
    const double lo1 = shd[0];
    g.sync();
    if (p < 0 || !(S > 0.0) || !isfinite(S)) {
      if (tid == 0) {
        atomicOr(a.flags + b, DSPARK_FLAG_NONFINITE);
        a.x_out[b * a.gamma + k] = 0;
        shi[1] = 0;
      }
    } else {
      // ---- level 2: the partition's stored logits, each thread a contiguous run of columns
      const int t0 = (int)((long long)p * a.ntiles / np), t1 = (int)((long long)(p + 1) * a.ntiles / np);
      const int tw = a.tile_chunks * kChunk;
      const int v0 = t0 * tw, n = min(t1 * tw, a.V) - v0;
      const float* row = a.ld + (size_t)k * a.sk + (size_t)b * a.sb + v0;
      const float inv_T = a.inv_T;
      auto w2 = [&](int j) -> double {
        const float z = __fmul_rn(__ldcg(row + j), inv_T);
        return z == -INFINITY ? 0.0 : (double)ex_shift(z, M);
      };
      const int e2 = (n + nth - 1) / nth;
      const int j0 = min(n, tid * e2), j1 = min(n, j0 + e2);
      double own2 = 0.0;
      for (int j = j0; j < j1; ++j) own2 += w2(j);
      double tot2 = 0.0;
      const double incl2 = lo1 + grp_incl_scan_d(own2, shs, g, tot2);
      const double excl2 = incl2 - own2;
      if (tid == 0) shi[1] = -1;
      g.sync();
      if (j0 < j1 && excl2 <= t && (t < incl2 || j1 == n)) {
        double R = excl2;
        int pick = -1, last = -1;
        double plo = 0.0, phi = 0.0;
        for (int j = j0; j < j1; ++j) {
          const double w = w2(j);
          if (w > 0.0) {
            last = j;
            if (t < R + w) {
              pick = j;
              plo = R;
              phi = R + w;
              break;
            }
          }
          R += w;
        }
        if (pick < 0 && last >= 0) {
          pick = last;
          plo = phi = t;  // rounding left u*S past the partition: a boundary, flagged
        }
        if (pick >= 0) {
          shi[1] = v0 + pick;
          uint32_t fl = 0;
          if ((t - plo) < 1e-6 * S || (phi - t) < 1e-6 * S) fl |= DSPARK_FLAG_DRAFT_NEAR_TIE;
          shi[2] = (int)fl;
        }
      }
      g.sync();
      if (tid == 0) {
        int x = shi[1];
        uint32_t fl = x >= 0 ? (uint32_t)shi[2] : (uint32_t)DSPARK_FLAG_NONFINITE;
        x = min(max(x, 0), a.V - 1);
        if (fl) atomicOr(a.flags + b, fl);
        a.x_out[b * a.gamma + k] = x;
        shi[1] = x;
      }
    }
    g.sync();
  }
  // the next step's B operand row: W1[x_k] (bf16 weights only)
  if (a.gbuf && k + 1 < a.gamma) {
    const int x = shi[1];
    const int cpr = a.r / 8;  // 16-byte chunks per row
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.W1) + (size_t)x * a.r);
    uint4* dst = reinterpret_cast<uint4*>(a.gbuf + (size_t)b * a.r);
    for (int c = tid; c < cpr; c += nth) dst[c] = __ldg(src + c);
  }
  g.sync();
}

// Combine of one request by one warp (the multi-step launch: the B requests' combines run on B
// warps spread over the grid, with no block barrier).  The same two levels and arithmetic as
// combine_group, each lane a contiguous run of records (level 1, np <= 256) or of logits
// (level 2).  The warp then copies W1[x_k] into row b of gbuf and adds 1 to *gready with
// release semantics.
__device__ void combine_warp(const DraftArgs& a, int k, int b, uint32_t* gready) {
  const size_t B = (size_t)a.B;
  const int np = a.np, lane = threadIdx.x & 31;
  constexpr unsigned FULL = 0xffffffffu;
  // requested before the first dependent load; greedy drafting takes no uniforms (u_draft may be null)
  const float u = a.greedy ? 0.f : __ldg(a.u_draft + b * a.gamma + k);
  int x = 0;
  uint32_t fl = 0;
  if (a.greedy) {
    Top2 t{-INFINITY, -1, -INFINITY};
    for (int p = lane; p < np; p += 32) {
      const ChunkStat s = ld_stat_cg(a.cpart + p * B + b);
      t = top2_merge(t, Top2{s.m, s.idx, s.m2});
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t = top2_merge(t, top2_shfl_xor(t, o));
    x = t.idx;
    if (x < 0 || x >= a.V) {
      fl |= DSPARK_FLAG_NONFINITE;
      x = min(max(x, 0), a.V - 1);
    }
    if (t.best - t.second <= 1e-6f * fmaxf(1.f, fabsf(t.best))) fl |= DSPARK_FLAG_DRAFT_NEAR_TIE;
  } else {
    // ---- level 1: each lane a contiguous run of at most 8 partition records
    const int e1 = (np + 31) / 32;
    const int i0 = min(np, lane * e1), i1 = min(np, i0 + e1);
    ChunkStat rec[8];
    float ml = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      rec[j] = (i0 + j < i1) ? ld_stat_cg(a.cpart + (size_t)(i0 + j) * B + b) : stat_empty();
      ml = fmaxf(ml, rec[j].m);
    }
    const float M = warp_max(ml);
    double w[8], own = 0.0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      w[j] = rec[j].m == -INFINITY ? 0.0 : (double)rec[j].s * (double)ex_shift(rec[j].m, M);
      own += w[j];
    }
    const double incl = warp_incl_scan_d(own);
    const double S = __shfl_sync(FULL, incl, 31);
    const double t = (double)u * S;
    const double excl = incl - own;
    int pick = -1;
    double plo = 0.0;
    if (i0 < i1 && excl <= t && (t < incl || i1 == np)) {
      double R = excl, lastlo = 0.0;
      int last = -1;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (pick < 0 && w[j] > 0.0) {
          last = i0 + j;
          lastlo = R;
          if (t < R + w[j]) {
            pick = i0 + j;
            plo = R;
          }
        }
        R += w[j];
      }
      if (pick < 0) {
        pick = last;
        plo = lastlo;
      }
    }
    const unsigned hit = __ballot_sync(FULL, pick >= 0);
    const int src = hit ? __ffs(hit) - 1 : 0;
    const int p = hit ? __shfl_sync(FULL, pick, src) : -1;
    const double lo1 = __shfl_sync(FULL, plo, src);
    if (p < 0 || !(S > 0.0) || !isfinite(S)) {
      fl |= DSPARK_FLAG_NONFINITE;
      x = 0;
    } else {
      // ---- level 2: the partition's stored logits in 128-column chunks (lane l holds quad l of
      // each chunk, so a chunk's lanes are in vocabulary order); every load of a block of 16
      // chunks is issued before any arithmetic (one L2 latency per 2048 columns)
      const int t0 = (int)((long long)p * a.ntiles / np), t1 = (int)((long long)(p + 1) * a.ntiles / np);
      const int tw = a.tile_chunks * kChunk;
      const int v0 = t0 * tw, n = min(t1 * tw, a.V) - v0;
      const float4* row4 = reinterpret_cast<const float4*>(a.ld + (size_t)k * a.sk + (size_t)b * a.sb + v0);  // 16-byte aligned
      const float inv_T = a.inv_T;
      const int nq4 = (n + 3) / 4;
      double base = lo1;  // weight before the current chunk
      int pk = -1, lastq = -1;
      double qlo = 0.0, qhi = 0.0;
      for (int blk = 0; blk < nq4 && pk < 0; blk += 16 * 32) {
        float4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int q = blk + 32 * i + lane;
          v[i] = q < nq4 ? __ldcg(row4 + q) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
        // weights of this lane's quads: element weight exp(z - M), 0 outside the partition
        auto quad_w = [&](const float4& q4, int e0, double (&we)[4]) -> double {
          const float l4[4] = {q4.x, q4.y, q4.z, q4.w};
          double wl = 0.0;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float z = __fmul_rn(l4[c], inv_T);
            we[c] = (e0 + c < n && z != -INFINITY) ? (double)ex_shift(z, M) : 0.0;
            wl += we[c];
          }
          return wl;
        };
        // chunk totals eight at a time: the eight butterflies interleave, and the chunk holding
        // u*S is found from the totals before any scan inside a chunk
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (pk >= 0 || blk + 32 * 8 * h >= nq4) break;  // warp-uniform
          double T[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            double we[4];
            T[i] = quad_w(v[8 * h + i], (blk + 32 * (8 * h + i) + lane) * 4, we);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int i = 0; i < 8; ++i) T[i] += __shfl_xor_sync(FULL, T[i], o);
          int cs = -1;
          double cbase = base;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (T[i] > 0.0) lastq = blk + 32 * (8 * h + i);  // a chunk with weight (refined below)
            if (cs < 0 && base + T[i] > t && T[i] > 0.0) {
              cs = i;
              cbase = base;
            }
            base += T[i];
          }
          if (cs >= 0) {
            // the chunk holds u*S: the first lane whose running sum passes it, then its element
            float4 vc = v[8 * h];
#pragma unroll
            for (int i = 1; i < 8; ++i)
              if (i == cs) vc = v[8 * h + i];
            const int e0 = (blk + 32 * (8 * h + cs) + lane) * 4;
            double we[4];
            const double wl = quad_w(vc, e0, we);
            const double incl2 = warp_incl_scan_d(wl);
            unsigned hitl = __ballot_sync(FULL, wl > 0.0 && cbase + incl2 > t);
            bool edge = false;
            if (!hitl) {  // the totals and the scan round differently: the chunk's last weight
              hitl = __ballot_sync(FULL, wl > 0.0);
              hitl = hitl ? (1u << (31 - __clz(hitl))) : 0u;
              edge = true;
            }
            if (hitl) {
              const int hl = __ffs(hitl) - 1;
              if (lane == hl) {
                double R = cbase + incl2 - wl;
                for (int c = 0; c < 4; ++c) {
                  if (!edge && we[c] > 0.0 && t < R + we[c]) {
                    pk = e0 + c;
                    qlo = R;
                    qhi = R + we[c];
                    break;
                  }
                  R += we[c];
                }
                if (pk < 0) {  // rounding inside the quad: its last element with weight
                  for (int c = 3; c >= 0 && pk < 0; --c)
                    if (we[c] > 0.0) pk = e0 + c;
                  qlo = qhi = t;
                }
              }
              pk = __shfl_sync(FULL, pk, hl);
              qlo = __shfl_sync(FULL, qlo, hl);
              qhi = __shfl_sync(FULL, qhi, hl);
            }
          }
        }
      }
      if (pk < 0 && lastq >= 0) {
        // rounding left u*S past the partition: the last quad with weight in the last chunk that
        // has any (one warp-wide pass over that chunk)
        const int q = lastq + lane;
        const float4 q4 = q < nq4 ? __ldcg(row4 + q) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        double we[4];
        const unsigned pos = __ballot_sync(FULL, [&] {
          const float l4[4] = {q4.x, q4.y, q4.z, q4.w};
          bool any = false;
          for (int c = 0; c < 4; ++c) {
            const float z = __fmul_rn(l4[c], inv_T);
            we[c] = (q * 4 + c < n && z != -INFINITY) ? (double)ex_shift(z, M) : 0.0;
            any |= we[c] > 0.0;
          }
          return any;
        }());
        lastq = pos ? lastq + 31 - __clz(pos) : -1;
      }
      if (pk < 0 && lastq >= 0) {
        // rounding left u*S past the partition: its last element with weight, flagged as a tie
        for (int c = 3; c >= 0 && pk < 0; --c) {
          const int e = lastq * 4 + c;
          if (e < n) {
            const float z = __fmul_rn(__ldcg(a.ld + (size_t)k * a.sk + (size_t)b * a.sb + v0 + e), inv_T);
            if (z != -INFINITY && ex_shift(z, M) > 0.f) pk = e;
          }
        }
        qlo = qhi = t;
      }
      if (pk >= 0) {
        x = v0 + pk;
        if ((t - qlo) < 1e-6 * S || (qhi - t) < 1e-6 * S) fl |= DSPARK_FLAG_DRAFT_NEAR_TIE;
      } else {
        fl |= DSPARK_FLAG_NONFINITE;
        x = 0;
      }
      x = min(max(x, 0), a.V - 1);
    }
  }
  if (lane == 0) {
    if (fl) atomicOr(a.flags + b, fl);
    a.x_out[b * a.gamma + k] = x;
  }
  // the next step's B operand row: W1[x_k] (bf16 weights only)
  if (a.gbuf && k + 1 < a.gamma) {
    const int cpr = a.r / 8;  // 16-byte chunks per row
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.W1) + (size_t)x * a.r);
    uint4* dst = reinterpret_cast<uint4*>(a.gbuf + (size_t)b * a.r);
    for (int c = lane; c < cpr; c += 32) dst[c] = __ldg(src + c);
    __syncwarp();  // orders the lanes' row stores before lane 0's release
    if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(gready) : "memory");
  }
}

// Combine kernel of the per-step launches: one CTA of kCombThreads per request.
constexpr int kCombThreads = 512;
__global__ void __launch_bounds__(kCombThreads) draft_combine(DraftArgs a, int k) {
  __shared__ double sh[72];
  pdl_trigger();
  pdl_wait();
  combine_group(a, k, blockIdx.x, Grp{(int)threadIdx.x, kCombThreads, -1}, sh);
}

// ============================================================================ host side

size_t draft_workspace_bytes(int B, int gamma, int V, int r) {
  (void)gamma;
  const size_t np_max = std::max<size_t>((size_t)(V + 255) / 256, 1024);  // partitions (either main pass)
  return kWsHeader + align_up((size_t)B * np_max * sizeof(ChunkStat), 256) + align_up((size_t)B * r * 2, 256);
}

size_t rnn_draft_workspace_bytes(int B, int gamma, int V, int r) {
  return draft_workspace_bytes(B, gamma, V, r) + align_up((size_t)B * r * 4, 256);
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
                     const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128 = true) {
  auto fn = encode_fn();
  if (!fn) return false;
  uint32_t es[3] = {1, 1, 1};
  CUresult rc = fn(m, dt, rank, base, dims, strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

template <typename K, typename... Args>
static cudaError_t launch_ex(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, bool coop,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (coop) {  // all CTAs resident at once (the launch fails otherwise)
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename WT, int BG>
static cudaError_t launch_fma(const DraftArgs& a, int k, cudaStream_t st, bool pdl) {
  const int vec_ok = (a.V % (int)(16 / sizeof(WT)) == 0 && (uintptr_t)a.W2 % 16 == 0) ? 1 : 0;
  const size_t smem = (size_t)(((BG * a.r + 3) & ~3) + 4 * BG * 256) * sizeof(float);
  auto kern = draft_main_fma<WT, BG>;
  const cudaError_t attr_rc = ensure_smem_attr((const void*)kern, smem);
  if (attr_rc != cudaSuccess) return attr_rc;
  dim3 grid((a.V + 255) / 256, (a.B + BG - 1) / BG);
  return launch_ex(kern, grid, dim3(128), smem, st, pdl, false, a, k, vec_ok);
}

template <typename WT>
static cudaError_t launch_fma_bg(const DraftArgs& a, int k, cudaStream_t st, bool pdl) {
  if (a.B <= 1) return launch_fma<WT, 1>(a, k, st, pdl);
  if (a.B <= 2) return launch_fma<WT, 2>(a, k, st, pdl);
  if (a.B <= 4) return launch_fma<WT, 4>(a, k, st, pdl);
  return launch_fma<WT, 8>(a, k, st, pdl);
}

static cudaError_t tc_set_smem(int nb, size_t smem) {
  return nb == 32 ? ensure_smem_attr((const void*)draft_main_tc<32>, smem)
                  : ensure_smem_attr((const void*)draft_main_tc<64>, smem);
}

dspark_status launch_draft(const DraftCall& c) {
  const Options opt = options();
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
  ld_strides(c.layout, c.B, c.gamma, c.V, a.sk, a.sb);
  a.rm = c.layout == DSPARK_REQUEST_MAJOR ? 1 : 0;
  a.spin_limit = opt.debug_wait_limit > 0 ? (uint32_t)std::min<long>(opt.debug_wait_limit, kSpinLimit) : kSpinLimit;
  a.barrier_extra = opt.debug_unreachable_barrier == 1 ? 1 : 0;
  a.B = c.B;
  a.gamma = c.gamma;
  a.V = c.V;
  a.r = c.r;
  a.nchunk = (c.V + kChunk - 1) / kChunk;
  a.cpart = reinterpret_cast<ChunkStat*>(static_cast<uint8_t*>(c.ws) + kWsHeader);
  {
    const size_t np_max = std::max<size_t>((size_t)(c.V + 255) / 256, 1024);
    uint8_t* gb = static_cast<uint8_t*>(c.ws) + kWsHeader + align_up((size_t)c.B * np_max * sizeof(ChunkStat), 256);
    a.gbuf = (c.w_dtype == DSPARK_BF16 && c.r % 64 == 0) ? reinterpret_cast<__nv_bfloat16*>(gb) : nullptr;
  }
  a.greedy = (c.T == 0.f) ? 1 : 0;
  a.inv_T = a.greedy ? 1.f : 1.f / c.T;
  const bool rnn = c.Wh != nullptr;
  if (rnn) {  // the recurrent head: CUDA-core pass, one state kernel before each step
    a.Wh = c.Wh;
    a.hstate = reinterpret_cast<float*>(static_cast<uint8_t*>(c.ws) + draft_workspace_bytes(c.B, c.gamma, c.V, c.r));
    a.h_out = c.h_out;
    a.gbuf = nullptr;
  }
  const bool pdl = opt.draft_pdl != 0 && !rnn;

  const bool aligned16 = ((uintptr_t)c.W1 % 16 == 0) && ((uintptr_t)c.W2 % 16 == 0) && ((uintptr_t)c.U % 16 == 0) &&
                         ((uintptr_t)c.ld_out % 16 == 0);
  const bool tc_ok = c.w_dtype == DSPARK_BF16 && c.r % 64 == 0 && c.r <= 256 && c.V % 8 == 0 && aligned16;
  bool use_tc = tc_ok && c.B >= opt.draft_tc_min_b && !rnn;
  if (opt.draft_force_path == 1) use_tc = false;
  if (opt.draft_force_path == 2 && !rnn) {
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

  CUtensorMap mW2, mU, mLd, mG;
  memset(&mG, 0, sizeof(mG));
  int n_bgroups = 1, cpg = 1, nb = 0;
  size_t tc_smem = 0;
  if (use_tc) {
    nb = c.B <= 32 ? 32 : 64;
    a.ntiles = (c.V + 63) / 64;  // half tiles: the unit of the CTAs' column shares
    a.tile_chunks = 64 / kChunk;
    n_bgroups = (c.B + nb - 1) / nb;
    const int sms = device_sm_count();
    cpg = std::max(1, sms / n_bgroups);
    cpg = std::min(cpg, a.ntiles);
    a.np = cpg;
    uint64_t dims[2] = {(uint64_t)c.V, (uint64_t)c.r};
    uint64_t strides[1] = {(uint64_t)c.V * 2};
    uint32_t box[2] = {64, (uint32_t)c.r};
    if (!make_map(&mW2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(c.W2), dims, strides, box)) {
      set_error("cuTensorMapEncodeTiled failed for W2");
      return DSPARK_ECUDA;
    }
    // A box is one 128-column tile of the nb requests of a group at one position (32 KB at
    // nb = 64: large copies keep the copy engine near full bandwidth, where 4 KB copies were
    // measured to stream at under half); position-major U / l_d [gamma][B][V]: dims {V, B, gamma}
    // request-major U / l_d: dims {V, gamma, B}, box {128, 1, nb} (the same [nb][128] layout in
    // shared memory; coordinates (column, k, b0))
    uint64_t udims[3] = {(uint64_t)c.V, (uint64_t)c.B, (uint64_t)c.gamma};
    uint64_t ustrides[2] = {(uint64_t)c.V * 4, (uint64_t)c.B * c.V * 4};
    uint32_t ubox[3] = {(uint32_t)kTcTile, (uint32_t)nb, 1};
    if (a.rm) {
      udims[1] = (uint64_t)c.gamma;
      udims[2] = (uint64_t)c.B;
      ustrides[1] = (uint64_t)c.gamma * c.V * 4;
      ubox[1] = 1;
      ubox[2] = (uint32_t)nb;
    }
    if (!make_map(&mU, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(c.U), udims, ustrides, ubox, false)) {
      set_error("cuTensorMapEncodeTiled failed for U");
      return DSPARK_ECUDA;
    }
    if (!make_map(&mLd, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, c.ld_out, udims, ustrides, ubox, false)) {
      set_error("cuTensorMapEncodeTiled failed for l_d");
      return DSPARK_ECUDA;
    }
    if (a.gbuf) {  // the B operand rows copied by the combine: [B][r] bf16, boxes of 64 x nb, 128-byte swizzle
      uint64_t gdims[2] = {(uint64_t)c.r, (uint64_t)c.B};
      uint64_t gstrides[1] = {(uint64_t)c.r * 2};
      uint32_t gbox[2] = {64, (uint32_t)nb};
      if (!make_map(&mG, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.gbuf, gdims, gstrides, gbox)) {
        set_error("cuTensorMapEncodeTiled failed for the B-operand rows");
        return DSPARK_ECUDA;
      }
    }
    tc_smem = tc_layout(c.r, nb).total + 1024;
    rc = tc_set_smem(nb, tc_smem);
    if (rc != cudaSuccess) {
      set_error(std::string("cudaFuncSetAttribute(draft_main_tc): ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  } else {
    a.ntiles = (c.V + 255) / 256;
    a.tile_chunks = 256 / kChunk;
    a.np = a.ntiles;
  }

  // the in-kernel combine takes <= 8 partition records a lane; other shapes run one launch pair
  // per step
  const bool fusable = a.np <= 256;
  if (use_tc && opt.draft_fused && fusable) {
    // all gamma steps in one cooperative launch (every CTA resident; grid barriers between steps)
    const dim3 grid(cpg * n_bgroups), block(kTcThreads);
    if (nb == 32)
      rc = launch_ex(draft_main_tc<32>, grid, block, tc_smem, c.stream, false, true, mW2, mU, mLd, mG, a, 0, c.gamma,
                     n_bgroups, cpg, 1);
    else
      rc = launch_ex(draft_main_tc<64>, grid, block, tc_smem, c.stream, false, true, mW2, mU, mLd, mG, a, 0, c.gamma,
                     n_bgroups, cpg, 1);
    if (rc == cudaSuccess) return DSPARK_OK;
    (void)cudaGetLastError();  // e.g. not all CTAs can be resident: one launch pair per step below
  }
  for (int k = 0; k < c.gamma; ++k) {
    // The first main pass waits for everything before the call in full: its producers read U
    // and W2 before the grid-dependency wait, which is only safe behind this call's own kernels.
    const bool pdl_k = pdl && k > 0;
    if (rnn) {
      const int thr = std::min(256, (c.r + 31) / 32 * 32);
      if (c.w_dtype == DSPARK_BF16)
        rnn_state_kernel<__nv_bfloat16><<<c.B, thr, (size_t)c.r * 4, c.stream>>>(a, k);
      else
        rnn_state_kernel<float><<<c.B, thr, (size_t)c.r * 4, c.stream>>>(a, k);
      rc = cudaGetLastError();
      if (rc != cudaSuccess) {
        set_error(std::string("recurrent state launch: ") + cudaGetErrorString(rc));
        return DSPARK_ECUDA;
      }
    }
    if (use_tc) {
      const dim3 grid(cpg * n_bgroups), block(kTcThreads);
      if (nb == 32)
        rc = launch_ex(draft_main_tc<32>, grid, block, tc_smem, c.stream, pdl_k, false, mW2, mU, mLd, mG, a, k, k + 1,
                       n_bgroups, cpg, 0);
      else
        rc = launch_ex(draft_main_tc<64>, grid, block, tc_smem, c.stream, pdl_k, false, mW2, mU, mLd, mG, a, k, k + 1,
                       n_bgroups, cpg, 0);
    } else if (c.w_dtype == DSPARK_BF16) {
      rc = launch_fma_bg<__nv_bfloat16>(a, k, c.stream, pdl_k);
    } else {
      rc = launch_fma_bg<float>(a, k, c.stream, pdl_k);
    }
    if (rc != cudaSuccess) {
      set_error(std::string("draft main pass launch: ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
    rc = launch_ex(draft_combine, dim3(c.B), dim3(kCombThreads), 0, c.stream, pdl, false, a, k);
    if (rc != cudaSuccess) {
      set_error(std::string("draft combine launch: ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  }
  return DSPARK_OK;
}

}  // namespace dspark
