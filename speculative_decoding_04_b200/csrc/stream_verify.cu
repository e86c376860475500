// Streaming verification: the rejection-sampling verify and the TV labels with every row of
// l_d and l_t read once from HBM and once more from L2, and no per-row barrier.
//
// [P1 "DeepSeek V4-Pro DSpark 推测解码方案深度解析" §大模型推理的显存瓶颈与推测解码的演进逻辑:
//  the target checks the drafted tokens left to right with rejection sampling, keeps the
//  longest passing prefix, resamples one token at the first failure and drops the rest]
// [P3 "DSpark Speculative Decoding", opening paragraph: longest consistent prefix + bonus token;
//  §Confidence-Scheduled Verification: label c*_k = 1 - ½‖p_d - p_t‖₁]
//
// Layout of the work.  A cluster of C CTAs takes rows (position k, request b) in turn; CTA r
// owns the r-th contiguous run of 1024-column tiles of every row.  Per row each CTA runs
//   P1  (tiles from HBM)  per-lane maxima and sums of 2^(z log2e - R) against an integer
//       reference R, so that every later rescaling is an exact power of two; the sums of l_t
//       per tile are kept for the bonus sample; the raw logits at the drafted token are kept;
//   --  the CTA's (R, S) pairs go to every CTA of the cluster (distributed shared memory and a
//       remote mbarrier arrive); each CTA folds them in rank order into the row's normalisers
//       log2 p = z log2e - K - lam (K an integer, lam in [0, 1)) and decides the acceptance;
//   P2  (the same tiles again, now from L2)  p_d, p_t, sum min(p_d, p_t) and
//       q = max(0, p_t - p_d) per tile (the residual sample's weights).
// The tiles of P1 of the next row sit between P1 and P2 of a row, so the exchange never
// stalls the tile pipeline, and a row's two reads are at most two rows of the whole grid
// apart (a few tens of MB against a 126 MB L2).
//
// Roles in a CTA of 320 threads: warps 0-7 consume tiles (tile g goes to warp g mod 8 and ring
// stage g mod 16), warp 8 issues the bulk copies, warp 9 combines partial results, exchanges
// them with the cluster, decides acceptance and writes the per-row records.  A small second
// kernel (one warp per request) finds n, samples the residual / bonus token by an inverse CDF
// over the per-tile weights and one rescanned tile, and writes y, n and c*.
// Every wait is bounded; after a timeout all roles stop and the status word is set.

#include <cooperative_groups.h>

#include <algorithm>
#include <cfloat>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dspark {

namespace {

constexpr int kSvTile = 1024;  // columns per tile
constexpr int kSvWarps = 8;    // consumer warps
constexpr int kSvStages = 16;  // ring stages of (l_d tile, l_t tile)
constexpr int kSvThreads = (kSvWarps + 2) * 32;
constexpr int kSvProducer = kSvWarps;
constexpr int kSvController = kSvWarps + 1;
constexpr int kSvPhaseSlots = 8;
constexpr int kSvJobSlots = 4;
constexpr int kSvMaxCluster = 8;
constexpr int kRNone = -(1 << 28);  // reference of an empty sum
constexpr int kRMax = 1 << 24;
constexpr size_t kSvRingBytes = (size_t)kSvStages * 2 * kSvTile * sizeof(float);

// A partial result: of a warp for one phase, or of a CTA for one row.
// P1: sd / st are sums of 2^(z log2e - rd / rt); P2: sd = sum min(p_d, p_t), st = sum q.
struct __align__(16) SvPart {
  double sd, st;
  int rd, rt;
  Top2 gd, gt;
  float ldx, ltx;  // raw logits at the drafted token (has_x)
  int has_x;
  uint32_t fl;
};

// Normalisers of a row: log2 p(v) = z(v) log2e - K - lam.
struct __align__(16) SvNorm {
  float Kd, lamd, Kt, lamt;
};

// Per-row record read by the finalize kernel.
struct __align__(16) SvRow {
  SvNorm nm;
  int acc;
  uint32_t fl;  // ACCEPT_NEAR_TIE / SAMPLE_NEAR_TIE
  int cand;     // greedy: argmax of l_t
  float cstar;  // greedy label
};

struct SvArgs {
  const float* ld;
  const float* lt;
  const int32_t* x;
  const int32_t* L;
  const float* u_acc;
  const float* u_res;
  int B, gamma, V, lt_rows, njobs, ntile, C;
  float inv_T;
  int greedy, do_verify;
  float* c_star;
  int32_t* n_acc;
  int32_t* y_out;
  uint32_t* flags;
  uint32_t* status;
  SvRow* rows;      // [B][gamma+1]
  double2* part;    // [B][gamma][C]: (sum min, sum q) of each CTA
  float2* trec;     // [B][gamma+1][ntile]: (R, s) of l_t per tile
  float* qrec;      // [B][gamma+1][ntile]: sum q per tile
};

struct SvJob {
  int b, k, rec;
  bool t, d, verify;
};

__device__ __forceinline__ SvJob sv_job(const SvArgs& a, int j) {
  SvJob J;
  J.k = j / a.B;
  J.b = j - J.k * a.B;
  J.rec = J.b * (a.gamma + 1) + J.k;
  int Lb = a.gamma;
  if (a.do_verify && a.L) Lb = min(max(__ldg(a.L + J.b), 0), a.gamma);
  const bool cstar = a.c_star != nullptr && J.k < a.gamma;
  J.verify = a.do_verify && J.k < Lb;
  const bool bonus = a.do_verify && J.k == Lb;
  J.d = cstar || (J.verify && !a.greedy);  // greedy acceptance needs only argmax l_t
  J.t = cstar || J.verify || bonus;
  return J;
}

// Next job of this cluster at or after j that reads anything; -1 when none is left.
__device__ __forceinline__ int sv_next(const SvArgs& a, int j, int ncl, SvJob& J) {
  for (; j < a.njobs; j += ncl) {
    J = sv_job(a, j);
    if (J.t) return j;
  }
  return -1;
}

__device__ __forceinline__ bool sv_p2(const SvArgs& a, const SvJob& J) { return !a.greedy && J.d; }

__device__ __forceinline__ float sv_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^d for integer d <= 0 (exact; 0 below the double range)
__device__ __forceinline__ double sv_pow2d(int d) {
  return d < -1022 ? 0.0 : __longlong_as_double((long long)(1023 + d) << 52);
}
__device__ __forceinline__ float sv_pow2f(int d) { return d < -126 ? 0.f : __int_as_float((127 + d) << 23); }

// Integer reference for a maximum m of z: R = ceil(m log2e), clamped; kRNone for an empty max.
__device__ __forceinline__ int sv_ref(float m) {
  if (!(m > -INFINITY)) return kRNone;
  const int R = __float2int_ru(m * kLog2e);
  return min(max(R, -kRMax), kRMax);
}

// (R, S) += (r, s) with exact power-of-two rescaling
__device__ __forceinline__ void sv_merge(int& R, double& S, int r, double s) {
  if (r > R) {
    S = S * sv_pow2d(R - r) + s;
    R = r;
  } else {
    S += s * sv_pow2d(r - R);
  }
}

__device__ __forceinline__ void sv_warp_ref_sum(int& R, double& S) {
  const int M = __reduce_max_sync(0xffffffffu, R);
  S = warp_sum_d(S * sv_pow2d(R - M));
  R = M;
}

// p_d and p_t of one column from its raw logits (shared by the second pass and the rescan
// in the finalize kernel, so that both see the same weights).
__device__ __forceinline__ void sv_probs(float ld, float lt, float inv_T, const SvNorm& n, float& pd, float& pt) {
  const float zd = __fmul_rn(ld, inv_T), zt = __fmul_rn(lt, inv_T);
  pd = sv_ex2(__fsub_rn(fmaf(zd, kLog2e, -n.Kd), n.lamd));
  pt = sv_ex2(__fsub_rn(fmaf(zt, kLog2e, -n.Kt), n.lamt));
}
__device__ __forceinline__ float sv_pt(float lt, float inv_T, const SvNorm& n) {
  return sv_ex2(__fsub_rn(fmaf(__fmul_rn(lt, inv_T), kLog2e, -n.Kt), n.lamt));
}

// Normalisers (K, lam) from (R, S): S = f 2^e with f in [0.5, 1), K = R + e - 1, lam = log2(2f).
__device__ __forceinline__ bool sv_norm(int R, double S, float& K, float& lam) {
  if (!(S > 0.0) || !(S <= DBL_MAX) || R == kRNone) {
    K = 0.f;
    lam = 0.f;
    return false;
  }
  int e = 0;
  const double f = frexp(S, &e);
  K = (float)(R + e - 1);
  lam = (float)log2(2.0 * f);
  return true;
}

__device__ __forceinline__ SvPart sv_empty_part() {
  SvPart p;
  p.sd = p.st = 0.0;
  p.rd = p.rt = kRNone;
  p.gd = Top2{-INFINITY, -1, -INFINITY};
  p.gt = Top2{-INFINITY, -1, -INFINITY};
  p.ldx = p.ltx = 0.f;
  p.has_x = 0;
  p.fl = 0;
  return p;
}

// Fold the partials held by lanes 0..n-1 of a warp (the other lanes hold empty partials);
// every lane returns the same result (each step is commutative, so the butterfly gives
// identical bits in all lanes and in every CTA that folds the same inputs).
__device__ __forceinline__ SvPart sv_fold(SvPart p, bool sums_are_plain) {
  SvPart r = p;
  if (sums_are_plain) {
    r.sd = warp_sum_d(p.sd);
    r.st = warp_sum_d(p.st);
  } else {
    sv_warp_ref_sum(r.rd, r.sd);
    sv_warp_ref_sum(r.rt, r.st);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    r.gd = top2_merge(r.gd, top2_shfl_xor(r.gd, o));
    r.gt = top2_merge(r.gt, top2_shfl_xor(r.gt, o));
  }
  const unsigned hx = __ballot_sync(0xffffffffu, p.has_x != 0);
  if (hx) {
    const int src = __ffs(hx) - 1;
    r.ldx = __shfl_sync(0xffffffffu, p.ldx, src);
    r.ltx = __shfl_sync(0xffffffffu, p.ltx, src);
    r.has_x = 1;
  } else {
    r.has_x = 0;
  }
  r.fl = __reduce_or_sync(0xffffffffu, p.fl);
  return r;
}

__device__ __forceinline__ bool sv_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Arrive on the mbarrier at the same shared-memory offset in CTA `rank` of the cluster; the
// release orders this thread's earlier stores into that CTA's shared memory before it.
__device__ __forceinline__ void sv_remote_arrive(uint64_t* bar, int rank) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
      "r"(rank)
      : "memory");
}

__device__ __forceinline__ void sv_cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct SvSync {
  volatile int* abort;
  uint32_t* status;
};

__device__ __forceinline__ bool sv_wait(const SvSync& s, uint64_t* bar, uint32_t parity, bool cluster_scope = false) {
  if (*s.abort) return false;
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (cluster_scope ? sv_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *s.abort) return false;
  }
  *s.abort = 1;
  atomicOr(s.status, (uint32_t)DSPARK_ETIMEOUT);
  return false;
}

__device__ __forceinline__ float f4c(const float4& v, int c) { return c == 0 ? v.x : (c == 1 ? v.y : (c == 2 ? v.z : v.w)); }

template <bool GREEDY>
__global__ void __launch_bounds__(kSvThreads, 1) verify_stream(SvArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / C, ncl = gridDim.x / C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ __align__(128) float ring[];  // [kSvStages][2][kSvTile]: l_d tile, l_t tile
  __shared__ __align__(8) uint64_t full[kSvStages], empty[kSvStages];
  __shared__ __align__(8) uint64_t phbar[kSvPhaseSlots];
  __shared__ __align__(8) uint64_t xbar[kSvJobSlots], dbar[kSvJobSlots];
  __shared__ SvPart wpart[kSvPhaseSlots][kSvWarps];
  __shared__ SvPart xs[kSvJobSlots][kSvMaxCluster];
  __shared__ SvNorm dec[kSvJobSlots];
  __shared__ int s_abort;

  const SvSync sy{&s_abort, a.status};
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSvStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kSvPhaseSlots; ++i) mbar_init(&phbar[i], kSvWarps);
    for (int i = 0; i < kSvJobSlots; ++i) {
      mbar_init(&xbar[i], C);
      mbar_init(&dbar[i], 1);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  sv_cluster_sync_all();  // peers' barriers are initialised before any remote arrive

  const int tb = (int)((long long)rank * a.ntile / C);
  const int nt = (int)((long long)(rank + 1) * a.ntile / C) - tb;  // tiles of this CTA per row (may be 0)
  const float inv_T = a.inv_T;

  if (warp == kSvProducer) {
    // ------------------------------------------------------------------ bulk copies
    if (lane == 0) {
      uint32_t G = 0;
      bool ok = true;
      auto issue = [&](const SvJob& J, bool with_d) {
        const float* rd = a.ld + ((size_t)J.k * a.B + J.b) * a.V;
        const float* rt = a.lt + ((size_t)J.b * a.lt_rows + J.k) * a.V;
        for (int t = 0; t < nt && ok; ++t) {
          const uint32_t g = G + t;
          const int s = (int)(g % kSvStages);
          if (!sv_wait(sy, &empty[s], ((g / kSvStages) & 1) ^ 1)) {
            ok = false;
            break;
          }
          const int v0 = (tb + t) * kSvTile;
          const uint32_t bytes = (uint32_t)min(kSvTile, a.V - v0) * 4u;
          float* st = ring + (size_t)s * 2 * kSvTile;
          mbar_arrive_expect_tx(&full[s], with_d ? 2 * bytes : bytes);
          if (with_d) bulk_g2s(st, rd + v0, bytes, &full[s]);
          bulk_g2s(st + kSvTile, rt + v0, bytes, &full[s]);
        }
        G += nt;
      };
      SvJob cur, prev;
      int j = sv_next(a, cid, ncl, cur);
      bool have_prev = false;
      while (ok) {
        const bool have_cur = j >= 0;
        if (have_cur) issue(cur, cur.d);
        if (have_prev && sv_p2(a, prev)) issue(prev, true);
        if (!have_cur) break;
        prev = cur;
        have_prev = true;
        j = sv_next(a, j + ncl, ncl, cur);
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        const uint32_t lo = G > (uint32_t)kSvStages ? G - kSvStages : 0u;
        for (uint32_t g = lo; g < G; ++g)
          for (uint32_t i = 0; i < kSpinLimit && !mbar_try_wait(&full[g % kSvStages], (g / kSvStages) & 1); ++i) {
          }
      }
    }
  } else if (warp == kSvController) {
    // ------------------------------------------------------------------ combine, exchange, decide
    int p = 0;
    bool ok = true;
    int xk_prev = -1, xk_cur = -1;
    float u_prev = 0.f, u_cur = 0.f;
    auto p1_end = [&](const SvJob& J, int i) {
      const int ps = p % kSvPhaseSlots;
      ok = sv_wait(sy, &phbar[ps], (p / kSvPhaseSlots) & 1);
      ++p;
      if (!ok) return;
      SvPart w = lane < kSvWarps ? wpart[ps][lane] : sv_empty_part();
      w = sv_fold(w, false);
      // push this CTA's partial into slot [i % 4][rank] of every CTA of the cluster
      if (lane < C) {
        SvPart* dst = cluster.map_shared_rank(&xs[i % kSvJobSlots][rank], lane);
        *dst = w;
        sv_remote_arrive(&xbar[i % kSvJobSlots], lane);
      }
      (void)J;
    };
    auto p2_end = [&](const SvJob& J) {
      const int ps = p % kSvPhaseSlots;
      ok = sv_wait(sy, &phbar[ps], (p / kSvPhaseSlots) & 1);
      ++p;
      if (!ok) return;
      SvPart w = lane < kSvWarps ? wpart[ps][lane] : sv_empty_part();
      const double sm = warp_sum_d(w.sd), sq = warp_sum_d(w.st);
      if (lane == 0 && J.k < a.gamma) a.part[((size_t)J.b * a.gamma + J.k) * C + rank] = make_double2(sm, sq);
    };
    SvJob cur, prev;
    int j = sv_next(a, cid, ncl, cur);
    bool have_prev = false;
    for (int i = 0; ok; ++i) {
      const bool have_cur = j >= 0;
      if (have_cur) {
        xk_cur = cur.verify ? __ldg(a.x + (size_t)cur.b * a.gamma + cur.k) : -1;
        u_cur = (cur.verify && !GREEDY) ? __ldg(a.u_acc + (size_t)cur.b * a.gamma + cur.k) : 0.f;
      }
      if (have_prev) {
        // ---- decide the previous row: fold the cluster's partials in rank order
        const int js = (i - 1) % kSvJobSlots;
        ok = sv_wait(sy, &xbar[js], ((i - 1) / kSvJobSlots) & 1, true);
        if (!ok) break;
        SvPart x = lane < C ? xs[js][lane] : sv_empty_part();
        x = sv_fold(x, false);
        SvRow row;
        row.acc = 0;
        row.fl = 0;
        row.cand = 0;
        row.cstar = 0.f;
        uint32_t dfl = x.fl;
        if (GREEDY) {
          row.nm = SvNorm{0.f, 0.f, 0.f, 0.f};
          const bool ttie = x.gt.best - x.gt.second <= 1e-6f * fmaxf(1.f, fabsf(x.gt.best));
          row.cand = min(max(x.gt.idx, 0), a.V - 1);
          if (x.gt.idx < 0) dfl |= DSPARK_FLAG_NONFINITE;
          row.cstar = (x.gd.idx == x.gt.idx) ? 1.f : 0.f;
          row.fl = ttie ? (DSPARK_FLAG_ACCEPT_NEAR_TIE | DSPARK_FLAG_SAMPLE_NEAR_TIE) : 0u;
          if (prev.verify) {
            if ((unsigned)xk_prev >= (unsigned)a.V) dfl |= DSPARK_FLAG_TOKEN_RANGE;
            row.acc = (xk_prev == x.gt.idx) ? 1 : 0;
          }
        } else {
          SvNorm nm;
          bool good = sv_norm(x.rt, x.st, nm.Kt, nm.lamt);
          if (prev.d) good &= sv_norm(x.rd, x.sd, nm.Kd, nm.lamd);
          else nm.Kd = nm.lamd = 0.f;
          if (!good) dfl |= DSPARK_FLAG_NONFINITE;
          row.nm = nm;
          if (lane == 0) dec[js] = nm;
          if (prev.verify) {
            if ((unsigned)xk_prev >= (unsigned)a.V || !x.has_x) {
              dfl |= DSPARK_FLAG_TOKEN_RANGE;
            } else {
              const double l2e = (double)kLog2e;
              const double zd = (double)__fmul_rn(x.ldx, inv_T), zt = (double)__fmul_rn(x.ltx, inv_T);
              const double pd = exp2(zd * l2e - (double)x.rd) / x.sd;
              const double pt = exp2(zt * l2e - (double)x.rt) / x.st;
              const double u = (double)u_prev;
              row.acc = (u * pd < pt) ? 1 : 0;
              if (pd > 0.0 && fabs(u - pt / pd) < 1e-6) row.fl |= DSPARK_FLAG_ACCEPT_NEAR_TIE;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&dbar[js]);  // the second pass of this row may start
        }
        if (rank == 0 && lane == 0) {
          a.rows[prev.rec] = row;
          if (dfl && a.flags) atomicOr(a.flags + prev.b, dfl);
        }
      }
      if (have_cur) {
        p1_end(cur, i);
        if (!ok) break;
      }
      if (have_prev && sv_p2(a, prev)) {
        p2_end(prev);
        if (!ok) break;
      }
      if (!have_cur) break;
      prev = cur;
      xk_prev = xk_cur;
      u_prev = u_cur;
      have_prev = true;
      j = sv_next(a, j + ncl, ncl, cur);
    }
  } else {
    // ------------------------------------------------------------------ tile consumers
    const int w = warp;
    uint32_t G = 0;
    int p = 0;
    bool ok = true;
    auto run_phase = [&](const SvJob& J, bool second, int i) {
      SvPart out = sv_empty_part();
      // first pass state (per lane)
      int Rd = kRNone, Rt = kRNone;
      double Sd = 0.0, St = 0.0;
      Top2 gd{-INFINITY, -1, -INFINITY}, gt{-INFINITY, -1, -INFINITY};
      uint32_t bad = 0;
      // second pass state
      double smin = 0.0, sq = 0.0;
      SvNorm nm{0.f, 0.f, 0.f, 0.f};
      const int xk = (!second && J.verify) ? __ldg(a.x + (size_t)J.b * a.gamma + J.k) : -1;
      if (second) {
        const int js = i % kSvJobSlots;
        ok = sv_wait(sy, &dbar[js], (i / kSvJobSlots) & 1);
        if (ok) nm = dec[js];
      }
      const bool with_d = second || J.d;
      const uint32_t g0 = G + (uint32_t)((w - (int)(G % kSvWarps) + kSvWarps) % kSvWarps);
      for (uint32_t g = g0; ok && g < G + (uint32_t)nt; g += kSvWarps) {
        const int t = (int)(g - G);
        const int s = (int)(g % kSvStages);
        if (!sv_wait(sy, &full[s], (g / kSvStages) & 1)) {
          ok = false;
          break;
        }
        const int v0 = (tb + t) * kSvTile;
        const int cnt = min(kSvTile, a.V - v0);
        const float* sd = ring + (size_t)s * 2 * kSvTile;
        const float* st = sd + kSvTile;
        float4 fd[8], ft[8];
        const float4 ninf = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int idx = (jj * 32 + lane) * 4;
          const bool v = idx < cnt;
          ft[jj] = v ? *reinterpret_cast<const float4*>(st + idx) : ninf;
          fd[jj] = (v && with_d) ? *reinterpret_cast<const float4*>(sd + idx) : ninf;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // the values are in registers
        if (!second) {
          // drafted token in this tile: keep its raw logits
          const int xi = xk - v0;
          if (xi >= 0 && xi < cnt && ((xi >> 2) & 31) == lane) {
            const int jj = xi >> 7, c = xi & 3;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (q == jj) {
                out.ldx = f4c(fd[q], c);
                out.ltx = f4c(ft[q], c);
              }
            out.has_x = 1;
          }
          if (GREEDY) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int base = v0 + (jj * 32 + lane) * 4;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const float vt = f4c(ft[jj], c), vd = f4c(fd[jj], c);
                bad |= (isnan(vt) || vt == INFINITY || isnan(vd) || vd == INFINITY) ? 1u : 0u;
                if (vt > -INFINITY) top2_push(gt, vt, base + c);
                if (with_d && vd > -INFINITY) top2_push(gd, vd, base + c);
              }
            }
          } else {
            float mt = -INFINITY, md = -INFINITY;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              ft[jj] = make_float4(__fmul_rn(ft[jj].x, inv_T), __fmul_rn(ft[jj].y, inv_T), __fmul_rn(ft[jj].z, inv_T),
                                   __fmul_rn(ft[jj].w, inv_T));
              mt = fmaxf(mt, fmaxf(fmaxf(ft[jj].x, ft[jj].y), fmaxf(ft[jj].z, ft[jj].w)));
              if (with_d) {
                fd[jj] = make_float4(__fmul_rn(fd[jj].x, inv_T), __fmul_rn(fd[jj].y, inv_T),
                                     __fmul_rn(fd[jj].z, inv_T), __fmul_rn(fd[jj].w, inv_T));
                md = fmaxf(md, fmaxf(fmaxf(fd[jj].x, fd[jj].y), fmaxf(fd[jj].z, fd[jj].w)));
              }
            }
            const int rt = sv_ref(mt);
            const float rtf = (float)rt;
            float stl = 0.f;
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              stl += (sv_ex2(fmaf(ft[jj].x, kLog2e, -rtf)) + sv_ex2(fmaf(ft[jj].y, kLog2e, -rtf))) +
                     (sv_ex2(fmaf(ft[jj].z, kLog2e, -rtf)) + sv_ex2(fmaf(ft[jj].w, kLog2e, -rtf)));
            bad |= (stl <= FLT_MAX) ? 0u : 1u;
            sv_merge(Rt, St, rt, (double)stl);
            if (a.do_verify) {
              // l_t weight of the tile for the bonus / fallback sample
              const int R = __reduce_max_sync(0xffffffffu, rt);
              const float sw = warp_sum_f(stl * sv_pow2f(rt - R));
              if (lane == 0) a.trec[(size_t)J.rec * a.ntile + tb + t] = make_float2((float)R, sw);
            }
            if (with_d) {
              const int rd = sv_ref(md);
              const float rdf = (float)rd;
              float sdl = 0.f;
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                sdl += (sv_ex2(fmaf(fd[jj].x, kLog2e, -rdf)) + sv_ex2(fmaf(fd[jj].y, kLog2e, -rdf))) +
                       (sv_ex2(fmaf(fd[jj].z, kLog2e, -rdf)) + sv_ex2(fmaf(fd[jj].w, kLog2e, -rdf)));
              bad |= (sdl <= FLT_MAX) ? 0u : 1u;
              sv_merge(Rd, Sd, rd, (double)sdl);
            }
          }
        } else {
          float sml = 0.f, ql = 0.f;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float pd, pt;
              sv_probs(f4c(fd[jj], c), f4c(ft[jj], c), inv_T, nm, pd, pt);
              const float mn = fminf(pd, pt);
              sml += mn;
              ql += pt - mn;
            }
          }
          smin += (double)sml;
          sq += (double)ql;
          if (J.verify) {
            const double qw = warp_sum_d((double)ql);
            if (lane == 0) a.qrec[(size_t)J.rec * a.ntile + tb + t] = (float)qw;
          }
        }
      }
      G += (uint32_t)nt;
      if (!ok) return;
      // ---- phase result of this warp
      if (!second) {
        if (GREEDY) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            gd = top2_merge(gd, top2_shfl_xor(gd, o));
            gt = top2_merge(gt, top2_shfl_xor(gt, o));
          }
          out.gd = gd;
          out.gt = gt;
        } else {
          sv_warp_ref_sum(Rd, Sd);
          sv_warp_ref_sum(Rt, St);
          out.rd = Rd;
          out.sd = Sd;
          out.rt = Rt;
          out.st = St;
        }
        const unsigned hx = __ballot_sync(0xffffffffu, out.has_x != 0);
        if (hx) {
          const int src = __ffs(hx) - 1;
          out.ldx = __shfl_sync(0xffffffffu, out.ldx, src);
          out.ltx = __shfl_sync(0xffffffffu, out.ltx, src);
          out.has_x = 1;
        }
        out.fl = __any_sync(0xffffffffu, bad != 0) ? (uint32_t)DSPARK_FLAG_NONFINITE : 0u;
      } else {
        out.sd = warp_sum_d(smin);
        out.st = warp_sum_d(sq);
      }
      const int ps = p % kSvPhaseSlots;
      if (lane == 0) {
        wpart[ps][w] = out;
        mbar_arrive(&phbar[ps]);
      }
      ++p;
    };
    SvJob cur, prev;
    int j = sv_next(a, cid, ncl, cur);
    bool have_prev = false;
    for (int i = 0; ok; ++i) {
      const bool have_cur = j >= 0;
      if (have_cur) run_phase(cur, false, i);
      if (ok && have_prev && sv_p2(a, prev)) run_phase(prev, true, i - 1);
      if (!have_cur) break;
      prev = cur;
      have_prev = true;
      j = sv_next(a, j + ncl, ncl, cur);
    }
  }

  __syncwarp();
  sv_cluster_sync_all();  // no CTA leaves while a peer may still write into its shared memory
}

// Inverse-CDF sample of row `rec` (one warp): weights q = max(0, p_t - p_d) when `resid`
// (falling back to p_t when their sum is 0), else p_t.  Tile weights come from the records of
// the main kernel; the tile holding u * W is rescanned element by element.
__device__ int sv_sample(const SvArgs& a, int b, int k, bool resid, const SvNorm& nm, uint32_t& fl) {
  const int lane = threadIdx.x & 31;
  const size_t rec = (size_t)b * (a.gamma + 1) + k;
  const float2* tr = a.trec + rec * a.ntile;
  const float* qr = a.qrec + rec * a.ntile;
  const int per = (a.ntile + 31) / 32;
  const int t_lo = min(lane * per, a.ntile), t_hi = min(t_lo + per, a.ntile);
  auto tile_w = [&](int t, bool use_q) -> double {
    if (use_q) return (double)qr[t];
    const float2 v = tr[t];  // (R, s): mass s * 2^(R - K_t - lam_t)
    return (double)v.y * exp2((double)v.x - (double)nm.Kt - (double)nm.lamt);
  };
  double own = 0.0;
  for (int t = t_lo; t < t_hi; ++t) own += tile_w(t, resid);
  double incl = warp_incl_scan_d(own);
  double W = __shfl_sync(0xffffffffu, incl, 31);
  if (resid) {
    if (W < 1e-3) fl |= DSPARK_FLAG_SMALL_RESIDUAL;
    if (!(W > 0.0)) {  // p_t == p_d up to rounding: the residual is empty, sample p_t
      resid = false;
      own = 0.0;
      for (int t = t_lo; t < t_hi; ++t) own += tile_w(t, false);
      incl = warp_incl_scan_d(own);
      W = __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  const double target = (double)__ldg(a.u_res + b) * W;
  // ---- tile holding the target
  unsigned m = __ballot_sync(0xffffffffu, incl > target);
  int c = 0;
  double P = 0.0;
  {
    int ln;
    bool last = false;
    if (m) {
      ln = __ffs(m) - 1;
    } else {  // u * W at or above the total through rounding: last tile with weight
      last = true;
      const unsigned pos = __ballot_sync(0xffffffffu, own > 0.0);
      ln = pos ? 31 - __clz(pos) : 0;
    }
    if (lane == ln) {
      double acc = incl - own;
      int pick = -1;
      double pick_P = acc;
      for (int t = t_lo; t < t_hi; ++t) {
        const double w = tile_w(t, resid);
        if (w > 0.0) {
          pick = t;
          pick_P = acc;
          if (!last && acc + w > target) break;
        }
        acc += w;
      }
      c = pick >= 0 ? pick : max(t_lo, 0);
      P = pick_P;
    }
    c = __shfl_sync(0xffffffffu, c, ln);
    P = __shfl_sync(0xffffffffu, P, ln);
  }
  c = min(max(c, 0), a.ntile - 1);
  // ---- rescan the tile: lane l takes columns v0 + 32 l .. v0 + 32 l + 31
  const int v0 = c * kSvTile;
  const int cnt = min(kSvTile, a.V - v0);
  const float* rowd = a.ld + ((size_t)k * a.B + b) * a.V + v0;
  const float* rowt = a.lt + ((size_t)b * a.lt_rows + k) * a.V + v0;
  float val[32];
  double lsum = 0.0;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int i = lane * 32 + e;
    float w = 0.f;
    if (i < cnt) {
      if (resid) {
        float pd, pt;
        sv_probs(rowd[i], rowt[i], a.inv_T, nm, pd, pt);
        w = pt - fminf(pd, pt);
      } else {
        w = sv_pt(rowt[i], a.inv_T, nm);
      }
    }
    val[e] = w;
    lsum += (double)w;
  }
  const double lincl = warp_incl_scan_d(lsum);
  const unsigned mm = __ballot_sync(0xffffffffu, P + lincl > target);
  int tok = -1;
  double lower = 0.0, upper = 0.0;
  if (mm) {
    const int ln = __ffs(mm) - 1;
    if (lane == ln) {
      double acc = P + lincl - lsum;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        if (tok < 0 && val[e] > 0.f && acc + (double)val[e] > target) {
          tok = v0 + lane * 32 + e;
          lower = acc;
          upper = acc + (double)val[e];
        }
        acc += (double)val[e];
      }
    }
    tok = __shfl_sync(0xffffffffu, tok, ln);
    lower = __shfl_sync(0xffffffffu, lower, ln);
    upper = __shfl_sync(0xffffffffu, upper, ln);
  }
  if (tok < 0) {  // rounding left the target past the tile: its last column with weight
    int lastv = -1;
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (val[e] > 0.f) lastv = v0 + lane * 32 + e;
    const unsigned pos = __ballot_sync(0xffffffffu, lastv >= 0);
    tok = pos ? __shfl_sync(0xffffffffu, lastv, 31 - __clz(pos)) : v0;
    lower = upper = target;
  }
  if (target - lower < 1e-6 * W || upper - target < 1e-6 * W) fl |= DSPARK_FLAG_SAMPLE_NEAR_TIE;
  return min(max(tok, 0), a.V - 1);
}

// n, y, c* and flags of every request (one warp per request).
__global__ void __launch_bounds__(128) verify_stream_finalize(SvArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * 4 + warp;
  if (b >= a.B) return;
  const int G = a.gamma, R = G + 1;
  const SvRow* rr = a.rows + (size_t)b * R;
  const int Lb = a.L ? min(max(__ldg(a.L + b), 0), G) : G;
  if (a.c_star) {
    for (int k = lane; k < G; k += 32) {
      float cs;
      if (a.greedy) {
        cs = rr[k].cstar;
      } else {
        double sm = 0.0, sq = 0.0;
        for (int r = 0; r < a.C; ++r) {
          const double2 v = a.part[((size_t)b * G + k) * a.C + r];
          sm += v.x;
          sq += v.y;
        }
        cs = (float)(sq <= 0.5 ? 1.0 - sq : sm);
      }
      a.c_star[(size_t)b * G + k] = cs;
    }
  }
  int n = Lb;
  for (int k0 = 0; k0 < Lb; k0 += 32) {
    const int k = k0 + lane;
    const unsigned m = __ballot_sync(0xffffffffu, k < Lb && !rr[k].acc);
    if (m) {
      n = k0 + __ffs(m) - 1;
      break;
    }
  }
  uint32_t fl = 0;
  for (int k = lane; k <= n && k < Lb; k += 32) fl |= rr[k].fl & DSPARK_FLAG_ACCEPT_NEAR_TIE;
  fl = __reduce_or_sync(0xffffffffu, fl);
  int tok;
  if (a.greedy) {
    tok = rr[n].cand;
    fl |= rr[n].fl & (DSPARK_FLAG_SAMPLE_NEAR_TIE | DSPARK_FLAG_SMALL_RESIDUAL);
  } else {
    tok = sv_sample(a, b, n, n < Lb, rr[n].nm, fl);
  }
  int32_t* y = a.y_out + (size_t)b * R;
  for (int j = lane; j < R; j += 32) y[j] = j < n ? a.x[(size_t)b * G + j] : (j == n ? tok : -1);
  if (lane == 0) {
    a.n_acc[b] = n;
    if (fl && a.flags) atomicOr(a.flags + b, fl);
  }
}

struct SvLayout {
  size_t rows, part, trec, qrec, total;
};

SvLayout sv_layout(int B, int gamma, int V) {
  const size_t R = (size_t)B * (gamma + 1);
  const size_t nt = (size_t)(V + kSvTile - 1) / kSvTile;
  SvLayout L;
  L.rows = kWsHeader;
  L.part = L.rows + align_up(R * sizeof(SvRow), 256);
  L.trec = L.part + align_up((size_t)B * gamma * kSvMaxCluster * sizeof(double2), 256);
  L.qrec = L.trec + align_up(R * nt * sizeof(float2), 256);
  L.total = L.qrec + align_up(R * nt * sizeof(float), 256);
  return L;
}

}  // namespace

size_t stream_verify_workspace_bytes(int B, int gamma, int V) { return sv_layout(B, gamma, V).total; }

// DSPARK_ENOTIMPL: this call is not for the streaming kernels (labels only, V not a multiple of
// 4, unaligned rows, a workspace sized for the per-row kernels, or no cluster fits).
dspark_status launch_verify_stream(const VerifyCall& c) {
  if (!c.do_verify || !options().verify_stream) return DSPARK_ENOTIMPL;
  if (c.V % 4 || (uintptr_t)c.ld % 16 || (uintptr_t)c.lt % 16) return DSPARK_ENOTIMPL;
  const SvLayout Ly = sv_layout(c.B, c.gamma, c.V);
  if (c.ws_bytes < Ly.total) return DSPARK_ENOTIMPL;
  int C = options().verify_stream_cluster;
  if (C != 1 && C != 2 && C != 4 && C != 8) C = 8;
  uint8_t* ws = static_cast<uint8_t*>(c.ws);
  SvArgs a{};
  a.ld = c.ld;
  a.lt = c.lt;
  a.x = c.x;
  a.L = c.L;
  a.u_acc = c.u_acc;
  a.u_res = c.u_res;
  a.B = c.B;
  a.gamma = c.gamma;
  a.V = c.V;
  a.lt_rows = c.lt_rows;
  a.njobs = c.B * (c.gamma + 1);
  a.ntile = (c.V + kSvTile - 1) / kSvTile;
  a.greedy = c.T == 0.f ? 1 : 0;
  a.inv_T = a.greedy ? 1.f : 1.f / c.T;
  a.do_verify = 1;
  a.c_star = c.c_star;
  a.n_acc = c.n_acc;
  a.y_out = c.y_out;
  a.flags = c.flags;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.rows = reinterpret_cast<SvRow*>(ws + Ly.rows);
  a.part = reinterpret_cast<double2*>(ws + Ly.part);
  a.trec = reinterpret_cast<float2*>(ws + Ly.trec);
  a.qrec = reinterpret_cast<float*>(ws + Ly.qrec);
  auto kern = a.greedy ? verify_stream<true> : verify_stream<false>;
  cudaError_t rc;
  static bool attr_set[2] = {false, false};
  if (!attr_set[a.greedy]) {
    rc = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSvRingBytes);
    if (rc != cudaSuccess) {
      set_error(std::string("cudaFuncSetAttribute(verify_stream): ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
    attr_set[a.greedy] = true;
  }
  rc = cudaMemsetAsync(ws, 0, kWsHeader, c.stream);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaMemsetAsync: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kSvThreads);
  cfg.dynamicSmemBytes = kSvRingBytes;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int ncl = 0;
  for (; C >= 1; C >>= 1) {
    attr[0].val.clusterDim.x = C;
    cfg.gridDim = dim3((unsigned)C);
    if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) == cudaSuccess && ncl > 0) break;
    (void)cudaGetLastError();
  }
  if (C < 1 || ncl <= 0) return DSPARK_ENOTIMPL;
  a.C = C;
  ncl = std::min(ncl, a.njobs);
  cfg.gridDim = dim3((unsigned)(ncl * C));
  rc = cudaLaunchKernelEx(&cfg, kern, a);
  if (rc != cudaSuccess) {
    set_error(std::string("verify_stream launch (cluster ") + std::to_string(C) + "): " + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  verify_stream_finalize<<<(c.B + 3) / 4, 128, 0, c.stream>>>(a);
  rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("verify_stream finalize launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

}  // namespace dspark
