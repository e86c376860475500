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
// owns the r-th contiguous run of 512-column tiles of every row.  With c = log2(e) / T every
// exponent is a = fma(l, c, -ref) in fp32 (l·c exact inside the fma).  Per row each CTA runs
//   P1  (tiles from HBM)  per-lane maxima and sums of 2^a against an integer reference, so that
//       every later rescaling is an exact power of two;
//   --  the CTA's (R, S) pairs go to every CTA of the cluster (st.async stores into distributed
//       shared memory that complete on the receiver's mbarrier); each CTA folds them into the
//       row's normalisers log2 p = l c - K - lam (K an integer, lam in [0, 1)) and decides the
//       acceptance;
//   P2  (the same tiles again, now from L2)  sum min(p_d, p_t), taken as one 2^x per column
//       with x = min(a_d - (lam_d - lam_t), a_t) and the factor 2^-lam_t applied per tile, and
//       whether any column has p_t > p_d (without one, q = 0 everywhere and the label is exactly
//       1); a rejection that may be its request's first also keeps sum q per tile,
//       q = p_t - min(p_d, p_t) (the residual sample's weights).
// The passes of a CTA form one stream of tiles (P1 of row i, then P2 of row i - lag, and so
// on) cut into ring stages of 16 tiles without regard to row boundaries, so a row's last
// stage is shared with the next pass and no consumer idles at the end of a row; the exchange
// sits between P1 and P2 of a row and never stalls the stream.  A row's two reads are at most
// a few rows of the whole grid apart (tens of MB against a 126 MB L2).
//
// Roles in a CTA of 608 threads: warp 16 streams the tiles through a 3-stage ring (per stage
// and pass one bulk copy of each row: copies of 4 KB were measured to cap the stream at under
// half the HBM bandwidth, 32 KB ones reach it); warps 0-15 each take one 512-column tile of a
// stage (the assignment rotates from stage to stage; the passes are latency-bound, and 16
// warps with 512 columns each measured faster than 8 with 1024); warp 17 folds the warps'
// partials and exchanges them with the cluster; warp 18 folds the cluster's partials, decides
// acceptance and writes the per-row records (two warps, so that a row's decision never waits
// behind the next row's exchange).
// A small second kernel (one warp per request) finds n, samples the residual / bonus token by
// an inverse CDF over the per-tile weights and one rescanned tile, and writes y, n and c*.
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

constexpr int kSvTile = 512;    // columns per tile (one consumer warp's piece of a stage)
constexpr int kSvWarps = 16;    // consumer warps (four per scheduler: the passes are latency-bound)
constexpr int kSvVec = kSvTile / 128;  // float4s per lane and row in a piece
constexpr int kSvBig = kSvWarps * kSvTile;          // columns per ring stage: one 32 KB copy per row
constexpr int kSvStages = 3;                         // ring stages of (l_d 8192 columns, l_t 8192 columns)
constexpr int kSvThreads = (kSvWarps + 3) * 32;
constexpr int kSvProducer = kSvWarps;
constexpr int kSvCombiner = kSvWarps + 1;
constexpr int kSvDecider = kSvWarps + 2;
constexpr int kSvPhaseSlots = 16;
constexpr int kSvJobSlots = 4;
constexpr int kSvMaxCluster = 16;
constexpr uint32_t kSvSuspendNs = 100000;            // longest single suspension of a waiting warp
constexpr uint64_t kSvTimeoutNs = 2000000000ull;     // a wait gives up after 2 s
constexpr int kRNone = -(1 << 28);  // reference of an empty sum
constexpr int kRMax = 1 << 24;
constexpr size_t kSvRingBytes = (size_t)kSvStages * 2 * kSvBig * sizeof(float);

// A partial result: of a warp for one phase, or of a CTA for one row.
// P1: sd / st are sums of 2^(z log2e - rd / rt); P2: sd = sum min(p_d, p_t), st = sum q.
struct __align__(16) SvPart {
  double sd, st;
  int rd, rt;
  Top2 gd, gt;
  float pad0, pad1;
  int pad2;
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
  int B, gamma, V, lt_rows, njobs, ntile, C, lag, l2hint;
  size_t ld_sk, ld_sb;  // element strides of the l_d row of position k and request b
  const int64_t* lt_off;  // flattened l_t: request b's rows start at row lt_off[b] (null: padded)
  long long lt_nrows;
  uint64_t wait_ns;  // bounded waits give up after this long
  int xbar_extra;    // test-only: partials the exchange barriers expect beyond the cluster
  float zscale;  // log2(e) / T (T > 0)
  int greedy, do_verify;
  float* c_star;
  int32_t* n_acc;
  int32_t* y_out;
  uint32_t* flags;
  uint32_t* status;
  int* rej;         // [B]: gamma + 1 - k of the earliest rejection seen so far (0: none)
  SvRow* rows;      // [B][gamma+1]
  double2* part;    // [B][gamma][C]: (sum min(p_d, p_t), warps that saw p_t > p_d) of each CTA
  float2* trec;     // [B][gamma+1][ntile]: (R, s) of l_t per tile (bonus rows)
  float* qrec;      // [B][gamma+1][ntile]: sum q per tile (rejected rows)
};

struct SvJob {
  int b, k, rec;
  bool t, d, verify, bonus;
};

__device__ __forceinline__ SvJob sv_job(const SvArgs& a, int j) {
  SvJob J;
  J.k = j / a.B;
  J.b = j - J.k * a.B;
  J.rec = J.b * (a.gamma + 1) + J.k;
  int Lb = a.gamma;
  if (a.do_verify && a.L) Lb = min(max(__ldg(a.L + J.b), 0), a.gamma);
  // a flattened l_t holds rows 0..L_b of a request only: labels exist there
  const bool cstar = a.c_star != nullptr && J.k < a.gamma && (!a.lt_off || J.k <= Lb);
  J.verify = a.do_verify && J.k < Lb;
  const bool bonus = a.do_verify && J.k == Lb;
  J.d = cstar || (J.verify && !a.greedy);  // greedy acceptance needs only argmax l_t
  J.t = cstar || J.verify || bonus;
  J.bonus = bonus;
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

// One phase of the tile stream: the first pass of a row, or its second pass.
struct SvPhase {
  SvJob J;
  bool second;
  int i;  // index of the row among this cluster's rows (exchange / decision slots)
};

// The phase sequence of a cluster with a lag of L rows (a.lag, 0 to 3): P1(row i) then
// P2(row i-L), for i = 0, 1, ..., until both have run out.  Every role walks the same sequence.
struct SvGen {
  int j, ncl, i, step, nrows, lag;
  bool exhausted;
  int r0, r1, r2, r3;  // job indices of rows i, i-1, i-2, i-3 (registers, not an indexed array)
  __device__ void init(const SvArgs& a, int cid, int ncl_) {
    ncl = ncl_;
    lag = a.lag;
    i = 0;
    step = 0;
    nrows = 0;
    exhausted = false;
    SvJob J;
    j = sv_next(a, cid, ncl, J);
    r0 = j;
    r1 = r2 = r3 = -1;
    if (j >= 0) nrows = 1;
    else exhausted = true;
  }
  __device__ bool next(const SvArgs& a, SvPhase& ph) {
    while (true) {
      if (step == 0) {
        step = 1;
        if (i < nrows) {
          ph.J = sv_job(a, r0);
          ph.second = false;
          ph.i = i;
          return true;
        }
      }
      if (step == 1) {
        step = 2;
        const int q = i - lag;
        if (q >= 0 && q < nrows) {
          const SvJob J = sv_job(a, lag == 0 ? r0 : (lag == 1 ? r1 : (lag == 2 ? r2 : r3)));
          if (sv_p2(a, J)) {
            ph.J = J;
            ph.second = true;
            ph.i = q;
            return true;
          }
        }
      }
      ++i;
      step = 0;
      r3 = r2;
      r2 = r1;
      r1 = r0;
      r0 = -1;
      if (!exhausted) {
        SvJob J;
        j = sv_next(a, j + ncl, ncl, J);
        if (j >= 0) {
          nrows = i + 1;
          r0 = j;
        } else {
          exhausted = true;
        }
      }
      if (exhausted && i - lag >= nrows) return false;
    }
  }
};

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

// Integer reference for a maximum m of the raw logits: R = ceil(m c), clamped; kRNone for an
// empty max.  With it every 2^fma(l, c, -R) of those logits is at most about 1.
__device__ __forceinline__ int sv_ref(float m, float c) {
  if (!(m > -INFINITY)) return kRNone;
  const int R = __float2int_ru(m * c);
  return min(max(R, -kRMax), kRMax);
}

// (R, S) += (r, s) in fp32 with exact power-of-two rescaling (lane sums across the tiles of a pass)
__device__ __forceinline__ void sv_merge_f(int& R, float& S, int r, float s) {
  const int M = max(R, r);
  S = fmaf(S, sv_pow2f(R - M), s * sv_pow2f(r - M));
  R = M;
}

__device__ __forceinline__ void sv_warp_ref_sum(int& R, double& S) {
  const int M = __reduce_max_sync(0xffffffffu, R);
  S = warp_sum_d(S * sv_pow2d(R - M));
  R = M;
}

// Same across the lanes of a warp for fp32 lane sums (32 terms, fp32 adds).
__device__ __forceinline__ void sv_warp_ref_sum_f(int& R, float& S) {
  const int M = __reduce_max_sync(0xffffffffu, R);
  S = warp_sum_f(S * sv_pow2f(R - M));
  R = M;
}

// Constants of the second pass of a row: x_d = fma(l_d, c, -K_d) - (lam_d - lam_t),
// x_t = fma(l_t, c, -K_t); then p_t = 2^x_t * 2^-lam_t and min(p_d, p_t) = 2^min(x_d, x_t) * 2^-lam_t.
struct SvP2 {
  float nkd, nkt, ndl;  // -K_d, -K_t, -(lam_d - lam_t)
  float scale;          // 2^-lam_t
};
__device__ __forceinline__ SvP2 sv_p2_consts(const SvNorm& n) {
  SvP2 k;
  k.nkd = -n.Kd;
  k.nkt = -n.Kt;
  k.ndl = -__fsub_rn(n.lamd, n.lamt);
  k.scale = (float)exp2(-(double)n.lamt);
  return k;
}
// Unscaled terms of one column (the second pass computes the same values two columns at a time
// with packed instructions, which round each element exactly like these).
__device__ __forceinline__ void sv_p2_terms(float ld, float lt, float c, const SvP2& k, float& pt, float& mn) {
  const float xd = __fadd_rn(fmaf(ld, c, k.nkd), k.ndl), xt = fmaf(lt, c, k.nkt);
  pt = sv_ex2(xt);
  mn = sv_ex2(fminf(xd, xt));
}
__device__ __forceinline__ float sv_pt_term(float lt, float c, const SvP2& k) { return sv_ex2(fmaf(lt, c, k.nkt)); }

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
  p.pad0 = p.pad1 = 0.f;
  p.pad2 = 0;
  p.fl = 0;
  return p;
}

// Fold the partials held by lanes 0..n-1 of a warp (the other lanes hold empty partials);
// every lane returns the same result (each step is commutative, so the butterfly gives
// identical bits in all lanes and in every CTA that folds the same inputs).
template <bool GREEDY>
__device__ __forceinline__ SvPart sv_fold(SvPart p) {
  SvPart r = p;
  if (GREEDY) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      r.gd = top2_merge(r.gd, top2_shfl_xor(r.gd, o));
      r.gt = top2_merge(r.gt, top2_shfl_xor(r.gt, o));
    }
  } else {
    sv_warp_ref_sum(r.rd, r.sd);
    sv_warp_ref_sum(r.rt, r.st);
  }
  r.fl = __reduce_or_sync(0xffffffffu, p.fl);
  return r;
}

// One wait on the phase with the given parity that suspends the warp until the phase completes
// or kSvSuspendNs pass (the hardware wakes it on completion), instead of polling in a loop.
__device__ __forceinline__ bool sv_try_wait_suspend(uint64_t* bar, uint32_t parity, bool cluster_scope) {
  uint32_t ok;
  if (cluster_scope)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSvSuspendNs)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSvSuspendNs)
        : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t sv_now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void sv_cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

struct SvSync {
  volatile int* abort;
  uint32_t* status;
  uint64_t limit_ns;  // a wait gives up after this long
};

// Bounded wait: gives up (setting the abort flag and the status word) after kSvTimeoutNs, or
// returns false at once when another role has given up.
__device__ __forceinline__ bool sv_wait(const SvSync& s, uint64_t* bar, uint32_t parity, bool cluster_scope = false) {
  if (*s.abort) return false;
  if (sv_try_wait_suspend(bar, parity, cluster_scope)) return true;
  const uint64_t t0 = sv_now_ns();
  while (true) {
    if (sv_try_wait_suspend(bar, parity, cluster_scope)) return true;
    if (*s.abort) return false;
    if (sv_now_ns() - t0 > s.limit_ns) break;
  }
  *s.abort = 1;
  atomicOr(s.status, (uint32_t)DSPARK_ETIMEOUT);
  return false;
}

// Bounded wait until a shared counter reaches `target` (counters written by another warp of
// the CTA), with a short sleep between polls.
__device__ __forceinline__ bool sv_wait_count(const SvSync& s, volatile int* cnt, int target) {
  if (*cnt >= target) return true;
  const uint64_t t0 = sv_now_ns();
  while (*cnt < target) {
    if (*s.abort) return false;
    if (sv_now_ns() - t0 > s.limit_ns) {
      *s.abort = 1;
      atomicOr(s.status, (uint32_t)DSPARK_ETIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

__device__ __forceinline__ float f4c(const float4& v, int c) { return c == 0 ? v.x : (c == 1 ? v.y : (c == 2 ? v.z : v.w)); }

// Packed fp32 pairs (sm_100): per element the same correctly rounded results as the scalar
// instructions, at half the instruction count.
__device__ __forceinline__ float2 f2add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
// max of three (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 lo2(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return make_float2(v.z, v.w); }

// fp32 sum of 2^fma(l, c, nR) over one lane's 16 values of a tile row (nR = minus a reference).
__device__ __forceinline__ float sv_lane_sum_at(const float4 (&v)[kSvVec], float c, float nR) {
  const float2 c2 = make_float2(c, c), nr2 = make_float2(nR, nR);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int jj = 0; jj < kSvVec; ++jj) {
    const float2 x = f2fma(lo2(v[jj]), c2, nr2), y = f2fma(hi2(v[jj]), c2, nr2);
    acc0 = f2add(acc0, make_float2(sv_ex2(x.x), sv_ex2(x.y)));
    acc1 = f2add(acc1, make_float2(sv_ex2(y.x), sv_ex2(y.y)));
  }
  const float2 acc = f2add(acc0, acc1);
  return acc.x + acc.y;
}

// First pass over one lane's 16 values of a tile row: the integer reference R of their maximum
// and the fp32 sum of 2^fma(l, c, -R).
__device__ __forceinline__ float sv_lane_sum(const float4 (&v)[kSvVec], float c, int& R) {
  float m = -INFINITY;
#pragma unroll
  for (int jj = 0; jj < kSvVec; ++jj) {
    m = fmax3(m, v[jj].x, v[jj].y);
    m = fmax3(m, v[jj].z, v[jj].w);
  }
  R = sv_ref(m, c);
  return sv_lane_sum_at(v, c, -(float)R);
}

// Adds one lane's tile row to the pass's running (R, S), nR = -R: against the reference that the
// lane's first tile of the pass set, or, when that sum reaches 2^100 or is not finite (a maximum
// far above the reference, or a non-finite logit), against the tile's own maximum with an exact
// power-of-two rescale.  Terms far below the reference flush to zero, 2^-125 or less of the sum.
// Returns the tile's sum; r is the reference it is taken against.
__device__ __forceinline__ float sv_lane_acc(const float4 (&v)[kSvVec], float c, int& R, float& nR, float& S,
                                             int& r) {
  if (R != kRNone) {
    const float s = sv_lane_sum_at(v, c, nR);
    if (s < 0x1p100f) {
      S += s;
      r = R;
      return s;
    }
  }
  const float s = sv_lane_sum(v, c, r);
  sv_merge_f(R, S, r, s);
  nR = -(float)R;
  return s;
}

// One consumer warp's tile of a stage (kSvTile columns of each row; `cnt` of them are real):
// lane l holds columns 4 (32 jj + l) .. + 3 of the tile in fd[jj] (l_d) and ft[jj] (l_t), -inf
// past `cnt`; without l_d, fd repeats ft.
__device__ __forceinline__ void sv_load_tile(const float* sd, const float* st, bool with_d, int cnt,
                                             float4 (&fd)[kSvVec], float4 (&ft)[kSvVec]) {
  const int lane = threadIdx.x & 31;
  if (cnt == kSvTile) {
#pragma unroll
    for (int jj = 0; jj < kSvVec; ++jj) {
      const int idx = (jj * 32 + lane) * 4;
      ft[jj] = *reinterpret_cast<const float4*>(st + idx);
      fd[jj] = with_d ? *reinterpret_cast<const float4*>(sd + idx) : ft[jj];
    }
  } else {
    const float4 ninf = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
#pragma unroll
    for (int jj = 0; jj < kSvVec; ++jj) {
      const int idx = (jj * 32 + lane) * 4;
      const bool v = idx < cnt;
      ft[jj] = v ? *reinterpret_cast<const float4*>(st + idx) : ninf;
      fd[jj] = (v && with_d) ? *reinterpret_cast<const float4*>(sd + idx) : ninf;
    }
  }
}

// First pass over one tile (T > 0): the lane sums of both rows against their references; for
// the bonus row (trec non-null) also the tile's l_t weight (R, s) for the bonus sample.
__device__ __forceinline__ void sv_p1_tile(const float4 (&fd)[kSvVec], const float4 (&ft)[kSvVec], float zc,
                                           bool with_d, float2* trec, int& Rd, float& Sd, float& nRd, int& Rt,
                                           float& St, float& nRt) {
  int rt;
  const float stl = sv_lane_acc(ft, zc, Rt, nRt, St, rt);
  if (trec) {
    const int R = __reduce_max_sync(0xffffffffu, rt);
    const float sw = warp_sum_f(stl * sv_pow2f(rt - R));
    if ((threadIdx.x & 31) == 0) *trec = make_float2((float)R, sw);
  }
  if (with_d) {
    int rd;
    sv_lane_acc(fd, zc, Rd, nRd, Sd, rd);
  }
}

// Second pass over one tile: 2^min(x_d, x_t) per column, unscaled, into smin and the max of
// x_t - x_d into dqmax (labels); a rejected row (needq) also stores its tile's sum of
// q = 2^x_t - 2^min(x_d, x_t), scaled, at *qrec.
__device__ __forceinline__ void sv_p2_tile(const float4 (&fd)[kSvVec], const float4 (&ft)[kSvVec], float zc,
                                           const SvP2& k2, bool needq, bool labels, float* qrec, float& smin,
                                           float& dqmax) {
  const float2 c2 = make_float2(zc, zc);
  const float2 nkd = make_float2(k2.nkd, k2.nkd), nkt = make_float2(k2.nkt, k2.nkt);
  const float2 ndl = make_float2(k2.ndl, k2.ndl), mone = make_float2(-1.f, -1.f);
  float2 sm2 = make_float2(0.f, 0.f);
  if (!needq) {
    if (labels) {
#pragma unroll
      for (int jj = 0; jj < kSvVec; ++jj) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float2 ld2 = h ? hi2(fd[jj]) : lo2(fd[jj]), lt2 = h ? hi2(ft[jj]) : lo2(ft[jj]);
          const float2 xd = f2add(f2fma(ld2, c2, nkd), ndl), xt = f2fma(lt2, c2, nkt);
          sm2 = f2add(sm2, make_float2(sv_ex2(fminf(xd.x, xt.x)), sv_ex2(fminf(xd.y, xt.y))));
          const float2 df = f2fma(xd, mone, xt);
          dqmax = fmax3(dqmax, df.x, df.y);
        }
      }
    }
  } else {
    float2 q2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int jj = 0; jj < kSvVec; ++jj) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 ld2 = h ? hi2(fd[jj]) : lo2(fd[jj]), lt2 = h ? hi2(ft[jj]) : lo2(ft[jj]);
        const float2 xd = f2add(f2fma(ld2, c2, nkd), ndl), xt = f2fma(lt2, c2, nkt);
        const float2 mn = make_float2(sv_ex2(fminf(xd.x, xt.x)), sv_ex2(fminf(xd.y, xt.y)));
        const float2 pt = make_float2(sv_ex2(xt.x), sv_ex2(xt.y));
        sm2 = f2add(sm2, mn);
        q2 = f2add(q2, f2fma(mn, mone, pt));
        const float2 df = f2fma(xd, mone, xt);
        dqmax = fmax3(dqmax, df.x, df.y);
      }
    }
    const float qw = warp_sum_f(q2.x + q2.y);
    if ((threadIdx.x & 31) == 0) *qrec = qw * k2.scale;
  }
  smin += sm2.x + sm2.y;
}

// Decision of a row for its second pass.
struct __align__(16) SvDec {
  SvNorm nm;
  int needq;  // rejected: the second pass also sums the residual weights q
  int pad0, pad1, pad2;
};

static_assert(sizeof(SvPart) == 64, "a partial is four 16-byte stores");

// Store a partial into the same shared-memory slot of CTA `rank` of the cluster with st.async,
// whose bytes count toward the transaction count of that CTA's mbarrier `bar` on arrival: the
// receiver's wait on the barrier then sees the data, and the sender needs no release fence
// (which would also wait for its earlier global stores).
__device__ __forceinline__ void sv_push_part(const SvPart& w, SvPart* slot, uint64_t* bar, int rank) {
  uint32_t ra, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(slot)), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(smem_u32(bar)), "r"(rank));
  const uint4* v = reinterpret_cast<const uint4*>(&w);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 x = v[q];
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                     ra + 16u * q),
                 "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w), "r"(rb)
                 : "memory");
  }
}

// Shared state of the combine and decide roles.
struct SvRoles {
  uint64_t* phbar;              // [kSvPhaseSlots]: the consumer warps' partials of a pass are in
  SvPart (*wpart)[kSvWarps];    // [kSvPhaseSlots][kSvWarps]
  SvPart (*xs)[kSvMaxCluster];  // [kSvJobSlots][C]: the cluster's partials of a row's first pass
  uint64_t* xbar;               // [kSvJobSlots]: all C partials of the row have arrived
  uint64_t* dbar;               // [kSvJobSlots]: the row is decided (dec[] complete)
  SvDec* dec;                   // [kSvJobSlots]
  volatile int* decided;        // rows of this cluster's sequence decided by this CTA
  volatile int* combined;       // passes whose warp partials the combiner has read
};

template <bool GREEDY>
__device__ __forceinline__ void sv_combine_role(const SvArgs& a, const SvSync& sy, const SvRoles& r, int C, int rank,
                                                int cid, int ncl) {
  const int lane = threadIdx.x & 31;
  // ------------------------------------------------------------------ combine and exchange
  // Per first pass: fold the warps' partials and push the CTA's into slot [i % 4][rank] of
  // every CTA of the cluster.  Per second pass: the CTA's label partials to global memory.
  // A push for row i waits until this CTA has decided row i-2: a peer that has decided row
  // i-2 has then seen this CTA's push of row i-2, so every peer has decided row i-4, the
  // previous user of the slot (the second passes give the same order when T > 0; greedy
  // verification has none).
  SvGen gen;
  gen.init(a, cid, ncl);
  SvPhase ph;
  int p = 0;
  bool ok = true;
  while (ok && gen.next(a, ph)) {
    const int ps = p % kSvPhaseSlots;
    ok = sv_wait(sy, &r.phbar[ps], (p / kSvPhaseSlots) & 1);
    ++p;
    if (!ok) break;
    SvPart w = lane < kSvWarps ? r.wpart[ps][lane] : sv_empty_part();
    // The count that frees the slot is stored after the shuffles that consume the slot's
    // values, so those reads are complete.  No fence here: one would also wait for this
    // warp's global stores of the previous pass, microseconds while the copies load HBM.
    if (!ph.second) {
      w = sv_fold<GREEDY>(w);
      if (lane == 0) *r.combined = p;
      const int i = ph.i;
      ok = sv_wait_count(sy, r.decided, i - 1);  // r.decided counts rows, so row i-2 is decided
      if (!ok) break;
      if (lane < C) sv_push_part(w, &r.xs[i % kSvJobSlots][rank], &r.xbar[i % kSvJobSlots], lane);
    } else {
      const double sm = warp_sum_d(w.sd), nq = warp_sum_d(w.st);
      if (lane == 0) *r.combined = p;
      if (lane == 0 && ph.J.k < a.gamma)
        a.part[((size_t)ph.J.b * a.gamma + ph.J.k) * C + rank] = make_double2(sm, nq);
    }
  }
}

template <bool GREEDY>
__device__ __forceinline__ void sv_decide_role(const SvArgs& a, const SvSync& sy, const SvRoles& r, int C, int rank,
                                               int cid, int ncl) {
  const int lane = threadIdx.x & 31;
  // ------------------------------------------------------------------ decide, row by row
  SvJob J;
  int j = sv_next(a, cid, ncl, J);
  bool ok = true;
  for (int i = 0; ok && j >= 0; ++i) {
    const int js = i % kSvJobSlots;
    // the drafted token and its uniform are requested before the wait for the peers
    // (and, for T > 0, the two logits at the drafted token)
    const int xk = J.verify ? __ldg(a.x + (size_t)J.b * a.gamma + J.k) : -1;
    const float u_acc = (J.verify && !GREEDY) ? __ldg(a.u_acc + (size_t)J.b * a.gamma + J.k) : 0.f;
    float ldx = 0.f, ltx = 0.f;
    if (!GREEDY && J.verify && (unsigned)xk < (unsigned)a.V) {
      ldx = __ldg(a.ld + (size_t)J.k * a.ld_sk + (size_t)J.b * a.ld_sb + xk);
      ltx = __ldg(a.lt + lt_row_index(a.lt_off, a.lt_nrows, a.lt_rows, J.b, J.k) * a.V + xk);
    }
    // the rejection record only grows: read before the wait, it can only ask for more residual
    // weights than needed, never fewer
    const int rej_seen = (!GREEDY && J.verify) ? __ldcg(a.rej + J.b) : 0;
    // the phase ends when this arrival is in and the cluster's C partials have landed
    if (lane == 0) mbar_arrive_expect_tx(&r.xbar[js], (uint32_t)((C + a.xbar_extra) * sizeof(SvPart)));
    ok = sv_wait(sy, &r.xbar[js], (i / kSvJobSlots) & 1, true);
    if (!ok) break;
    SvPart x = lane < C ? r.xs[js][lane] : sv_empty_part();
    x = sv_fold<GREEDY>(x);
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
      if (J.verify) {
        if ((unsigned)xk >= (unsigned)a.V) dfl |= DSPARK_FLAG_TOKEN_RANGE;
        row.acc = (xk == x.gt.idx) ? 1 : 0;
      }
    } else {
      SvNorm nm;
      bool good = sv_norm(x.rt, x.st, nm.Kt, nm.lamt);
      if (J.d) good &= sv_norm(x.rd, x.sd, nm.Kd, nm.lamd);
      else nm.Kd = nm.lamd = 0.f;
      if (!good) dfl |= DSPARK_FLAG_NONFINITE;
      row.nm = nm;
      if (J.verify) {
        if ((unsigned)xk >= (unsigned)a.V) {
          dfl |= DSPARK_FLAG_TOKEN_RANGE;
        } else {
          // u p_d(x) < p_t(x) with p = 2^(l c - R) / S, in fp64 (l c is exact there)
          const double pd = exp2((double)ldx * (double)a.zscale - (double)x.rd) / x.sd;
          const double pt = exp2((double)ltx * (double)a.zscale - (double)x.rt) / x.st;
          const double u = (double)u_acc;
          row.acc = (u * pd < pt) ? 1 : 0;
          if (pd > 0.0 && fabs(u - pt / pd) < 1e-6) row.fl |= DSPARK_FLAG_ACCEPT_NEAR_TIE;
        }
      }
      // residual weights only for a rejection that may be the request's first (the others are
      // never sampled); a rejection is published for the deciders of later rows
      const int enc = a.gamma + 1 - J.k;
      const bool rej = J.verify && !row.acc;
      const bool needq = rej && rej_seen <= enc;
      if (lane == 0) r.dec[js] = SvDec{nm, needq ? 1 : 0, 0, 0, 0};
      if (rej && rank == 0 && lane == 0) atomicMax(a.rej + J.b, enc);
      __syncwarp();
      if (lane == 0) mbar_arrive(&r.dbar[js]);  // the second pass of this row may start
    }
    if (rank == 0 && lane == 0) {
      a.rows[J.rec] = row;
      if (dfl && a.flags) atomicOr(a.flags + J.b, dfl);
    }
    // the count that frees this row's slots follows the shuffles that consumed them (no fence:
    // it would wait for the row's global stores above)
    __syncwarp();
    if (lane == 0) *r.decided = i + 1;
    j = sv_next(a, j + ncl, ncl, J);
  }
}

template <bool GREEDY>
__global__ void __launch_bounds__(kSvThreads, 1) verify_stream(SvArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / C, ncl = gridDim.x / C;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  extern __shared__ __align__(128) float ring[];  // [kSvStages][2][kSvBig]: l_d columns, l_t columns
  __shared__ __align__(8) uint64_t full[kSvStages], empty[kSvStages];
  __shared__ __align__(8) uint64_t phbar[kSvPhaseSlots];
  __shared__ __align__(8) uint64_t xbar[kSvJobSlots], dbar[kSvJobSlots];
  __shared__ SvPart wpart[kSvPhaseSlots][kSvWarps];
  __shared__ SvPart xs[kSvJobSlots][kSvMaxCluster];
  __shared__ SvDec dec[kSvJobSlots];
  __shared__ int s_abort;
  __shared__ volatile int s_decided;  // rows of this cluster's sequence decided by this CTA
  __shared__ volatile int s_combined;  // passes whose warp partials the combiner has read

  const SvSync sy{&s_abort, a.status, a.wait_ns};
  const SvRoles roles{phbar, wpart, xs, xbar, dbar, dec, &s_decided, &s_combined};
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSvStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kSvWarps);
    }
    for (int i = 0; i < kSvPhaseSlots; ++i) mbar_init(&phbar[i], kSvWarps);
    for (int i = 0; i < kSvJobSlots; ++i) {
      mbar_init(&xbar[i], 1);  // the decider's arrival; the partials count as transaction bytes
      mbar_init(&dbar[i], 1);
    }
    s_abort = 0;
    s_decided = 0;
    s_combined = 0;
    fence_mbar_init();
  }
  __syncthreads();
  sv_cluster_sync_all();  // peers' barriers are initialised before any remote store completes on them

  // This CTA's segment of every row: tiles tb .. tb + nt - 1.  Pass number p of the CTA's
  // sequence covers tiles p*nt .. p*nt + nt - 1 of the CTA's tile stream; stage g of the ring
  // holds stream tiles 16g .. 16g + 15.
  const int tb = (int)((long long)rank * a.ntile / C);
  const int nt = (int)((long long)(rank + 1) * a.ntile / C) - tb;  // may be 0
  const float zc = a.zscale;

  if (warp == kSvProducer) {
    // ------------------------------------------------------------------ bulk copies
    if (lane == 0) {
      const uint64_t pol_last = l2_policy_evict_last(), pol_first = l2_policy_evict_first();
      SvGen gen;
      gen.init(a, cid, ncl);
      SvPhase ph;
      bool have = nt > 0 && gen.next(a, ph);
      int pbase = 0;  // first stream tile of the pass ph
      uint32_t g = 0;
      bool ok = true;
      for (; have; ++g) {
        const int s = (int)(g % kSvStages);
        if (!sv_wait(sy, &empty[s], ((g / kSvStages) & 1) ^ 1)) {
          ok = false;
          break;
        }
        const int T0 = (int)g * kSvWarps, T1 = T0 + kSvWarps;
        float* stg = ring + (size_t)s * 2 * kSvBig;
        // one copy per row for each pass that has tiles in this stage
        while (have && pbase < T1) {
          const int lo = max(T0, pbase), hi = min(T1, pbase + nt);
          const int c0 = (tb + lo - pbase) * kSvTile, c1 = min((tb + hi - pbase) * kSvTile, a.V);
          const uint32_t bytes = (uint32_t)(c1 - c0) * 4u;
          const bool with_d = ph.second || ph.J.d;
          const float* rd = a.ld + (size_t)ph.J.k * a.ld_sk + (size_t)ph.J.b * a.ld_sb;
          const float* rt = a.lt + lt_row_index(a.lt_off, a.lt_nrows, a.lt_rows, ph.J.b, ph.J.k) * a.V;
          mbar_expect_tx(&full[s], with_d ? 2 * bytes : bytes);
          if (a.l2hint) {
            // first pass: keep the lines for the second; second pass: they are done with
            const uint64_t pol = (ph.second || !sv_p2(a, ph.J)) ? pol_first : pol_last;
            if (with_d) bulk_g2s_hint(stg + (lo - T0) * kSvTile, rd + c0, bytes, &full[s], pol);
            bulk_g2s_hint(stg + kSvBig + (lo - T0) * kSvTile, rt + c0, bytes, &full[s], pol);
          } else {
            if (with_d) bulk_g2s(stg + (lo - T0) * kSvTile, rd + c0, bytes, &full[s]);
            bulk_g2s(stg + kSvBig + (lo - T0) * kSvTile, rt + c0, bytes, &full[s]);
          }
          if (hi < pbase + nt) break;  // the pass goes on in the next stage
          have = gen.next(a, ph);
          pbase += nt;
        }
        mbar_arrive(&full[s]);
      }
      if (!ok) {
        // let the copies still in flight land before the CTA can exit
        const uint32_t lo = g > (uint32_t)kSvStages ? g - kSvStages : 0u;
        for (uint32_t gb = lo; gb < g; ++gb)
          for (uint32_t i = 0; i < kSpinLimit && !mbar_try_wait(&full[gb % kSvStages], (gb / kSvStages) & 1); ++i) {
          }
      }
    }
  } else if (warp == kSvCombiner) {
    sv_combine_role<GREEDY>(a, sy, roles, C, rank, cid, ncl);
  } else if (warp == kSvDecider) {
    sv_decide_role<GREEDY>(a, sy, roles, C, rank, cid, ncl);
  } else {
    // ------------------------------------------------------------------ tile consumers
    const int w = warp;
    const int last_tile = a.ntile - 1 - tb;  // the segment's ragged tile, if it has it
    const int last_cnt = a.V - (a.ntile - 1) * kSvTile;
    bool ok = true;
    int p = 0;  // passes finished by this warp (slot of the partials)
    // state of the current pass
    int Rd = kRNone, Rt = kRNone;
    float Sd = 0.f, St = 0.f, nRd = 0.f, nRt = 0.f;
    Top2 gd{-INFINITY, -1, -INFINITY}, gt{-INFINITY, -1, -INFINITY};
    uint32_t bad = 0;
    float smin = 0.f;       // second pass: unscaled sum of 2^min(x_d, x_t)
    float dqmax = -INFINITY;  // second pass: max of x_t - x_d (> 0: some column has p_t > p_d)
    SvP2 k2{0.f, 0.f, 0.f, 1.f};
    bool needq = false;

    SvGen cgen;
    cgen.init(a, cid, ncl);
    SvPhase ph{};
    auto start = [&]() {
      Rd = Rt = kRNone;
      Sd = St = 0.f;
      gd = Top2{-INFINITY, -1, -INFINITY};
      gt = Top2{-INFINITY, -1, -INFINITY};
      bad = 0;
      smin = 0.f;
      dqmax = -INFINITY;
      if (ph.second) {
        const int js = ph.i % kSvJobSlots;
        ok = __all_sync(0xffffffffu, sv_wait(sy, &dbar[js], (ph.i / kSvJobSlots) & 1));
        if (ok) {
          const SvDec dd = dec[js];
          k2 = sv_p2_consts(dd.nm);
          needq = dd.needq != 0;
        }
      }
    };
    auto finish = [&]() {
      SvPart out = sv_empty_part();
      if (!ph.second) {
        if (GREEDY) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            gd = top2_merge(gd, top2_shfl_xor(gd, o));
            gt = top2_merge(gt, top2_shfl_xor(gt, o));
          }
          out.gd = gd;
          out.gt = gt;
        } else {
          bad |= (St <= FLT_MAX && Sd <= FLT_MAX) ? 0u : 1u;  // a non-finite logit of the pass
          sv_warp_ref_sum_f(Rd, Sd);
          sv_warp_ref_sum_f(Rt, St);
          out.rd = Rd;
          out.sd = (double)Sd;
          out.rt = Rt;
          out.st = (double)St;
        }
        out.fl = __any_sync(0xffffffffu, bad != 0) ? (uint32_t)DSPARK_FLAG_NONFINITE : 0u;
      } else {
        out.sd = (double)warp_sum_f(smin) * (double)k2.scale;
        out.st = __any_sync(0xffffffffu, dqmax > 0.f) ? 1.0 : 0.0;
      }
      const int ps = p % kSvPhaseSlots;
      // the slot's previous pass (p - 16) must have been read: without a pass that waits for a
      // decision (greedy verification, or a CTA whose segment is empty) nothing else bounds
      // how far the warps run ahead of the combiner
      ok = __all_sync(0xffffffffu, sv_wait_count(sy, &s_combined, p - kSvPhaseSlots + 1));
      if (!ok) return;
      if (lane == 0) {
        wpart[ps][w] = out;
        mbar_arrive(&phbar[ps]);
      }
      ++p;
    };

    bool have = cgen.next(a, ph);
    if (have) start();
    int pbase = 0;
    for (uint32_t g = 0; ok && have; ++g) {
      const int q = (w + (int)g) & (kSvWarps - 1);  // slot of this warp in stage g
      const int T = (int)g * kSvWarps + q;
      while (T >= pbase + nt) {  // passes that end before this tile
        finish();
        if (!ok) break;
        have = cgen.next(a, ph);
        pbase += nt;
        if (!have) break;
        start();
        if (!ok) break;
      }
      if (!have || !ok) break;
      const int s = (int)(g % kSvStages);
      if (!__all_sync(0xffffffffu, sv_wait(sy, &full[s], (g / kSvStages) & 1))) {
        ok = false;
        break;
      }
      const int t = T - pbase;  // tile of this CTA's segment
      const int v0 = (tb + t) * kSvTile;
      const float* sd = ring + (size_t)s * 2 * kSvBig + q * kSvTile;
      const float* st = sd + kSvBig;
      const bool with_d = ph.second || ph.J.d;
      float4 fd[kSvVec], ft[kSvVec];
      sv_load_tile(sd, st, with_d, t == last_tile ? last_cnt : kSvTile, fd, ft);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // the values are in registers
      if (!ph.second) {
        if (GREEDY) {
#pragma unroll
          for (int jj = 0; jj < kSvVec; ++jj) {
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
          sv_p1_tile(fd, ft, zc, with_d, ph.J.bonus ? a.trec + (size_t)ph.J.rec * a.ntile + tb + t : nullptr, Rd, Sd,
                     nRd, Rt, St, nRt);
        }
      } else {
        sv_p2_tile(fd, ft, zc, k2, needq, a.c_star != nullptr, needq ? a.qrec + (size_t)ph.J.rec * a.ntile + tb + t : nullptr,
                   smin, dqmax);
      }
    }
  }

  __syncwarp();
  sv_cluster_sync_all();  // no CTA leaves while a peer may still write into its shared memory
}

// Inverse-CDF sample of row `rec` (one warp): weights q = max(0, p_t - p_d) when `resid`
// (falling back to p_t when their sum is 0), else p_t.  Tile weights come from the records of
// the main kernel (q of a rejected row, p_t of the bonus row); the p_t fallback of a rejected
// row, which only an empty residual reaches, sums its tiles here.  The tile holding u * W is
// rescanned element by element with the second pass's arithmetic.
__device__ int sv_sample(const SvArgs& a, int b, int k, bool resid, const SvNorm& nm, uint32_t& fl) {
  const int lane = threadIdx.x & 31;
  const size_t rec = (size_t)b * (a.gamma + 1) + k;
  const float2* tr = a.trec + rec * a.ntile;
  const float* qr = a.qrec + rec * a.ntile;
  const bool has_trec = !resid;  // the bonus row
  const SvP2 k2 = sv_p2_consts(nm);
  const float zc = a.zscale;
  const float* rowd = a.ld + (size_t)k * a.ld_sk + (size_t)b * a.ld_sb;
  const float* rowt = a.lt + lt_row_index(a.lt_off, a.lt_nrows, a.lt_rows, b, k) * a.V;
  const int per = (a.ntile + 31) / 32;
  const int t_lo = min(lane * per, a.ntile), t_hi = min(t_lo + per, a.ntile);
  auto tile_w = [&](int t, bool use_q) -> double {
    if (use_q) return (double)qr[t];
    if (has_trec) {
      const float2 v = tr[t];  // (R, s): mass s * 2^(R - K_t - lam_t)
      return (double)v.y * exp2((double)v.x - (double)nm.Kt - (double)nm.lamt);
    }
    double sum = 0.0;
    for (int v = t * kSvTile, e = min(v + kSvTile, a.V); v < e; ++v) sum += (double)(sv_pt_term(rowt[v], zc, k2) * k2.scale);
    return sum;
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
  float val[32];
  double lsum = 0.0;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int i = lane * 32 + e;
    float w = 0.f;
    if (i < cnt) {
      if (resid) {
        float pt, mn;
        sv_p2_terms(rowd[v0 + i], rowt[v0 + i], zc, k2, pt, mn);
        w = __fmul_rn(__fsub_rn(pt, mn), k2.scale);
      } else {
        w = __fmul_rn(sv_pt_term(rowt[v0 + i], zc, k2), k2.scale);
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
  const bool timed_out = __ldcg(a.status) != 0u;
  if (a.c_star) {
    for (int k = lane; k < G; k += 32) {
      float cs;
      if (a.lt_off && k > Lb) {
        cs = __int_as_float(0x7fc00000);  // no target row in the flattened block: NaN
      } else if (a.greedy) {
        cs = rr[k].cstar;
      } else {
        // sum min(p_d, p_t); exactly 1 when no column has p_t > p_d (then q = 0 everywhere)
        double sm = 0.0, nq = 0.0;
        for (int r = 0; r < a.C; ++r) {
          const double2 v = a.part[((size_t)b * G + k) * a.C + r];
          sm += v.x;
          nq += v.y;
        }
        cs = nq > 0.0 ? (float)fmin(sm, 1.0) : 1.f;
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
  if (timed_out) fl |= DSPARK_FLAG_DEVICE_TIMEOUT;
  if (a.lt_off && ragged_mismatch(a.lt_off, a.lt_nrows, b, Lb)) fl |= DSPARK_FLAG_RAGGED_OFFSETS;
  int32_t* y = a.y_out + (size_t)b * R;
  for (int j = lane; j < R; j += 32) y[j] = j < n ? a.x[(size_t)b * G + j] : (j == n ? tok : -1);
  if (lane == 0) {
    a.n_acc[b] = n;
    if (fl && a.flags) atomicOr(a.flags + b, fl);
  }
}

struct SvLayout {
  size_t rej, rows, part, trec, qrec, total;
};

SvLayout sv_layout(int B, int gamma, int V) {
  const size_t R = (size_t)B * (gamma + 1);
  const size_t nt = (size_t)(V + kSvTile - 1) / kSvTile;
  SvLayout L;
  L.rej = kWsHeader;
  L.rows = L.rej + align_up((size_t)B * sizeof(int), 256);
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
  const Options opt = options();
  if (!c.do_verify || c.per_row_only || opt.verify_impl != 0) return DSPARK_ENOTIMPL;
  if (c.V % 4 || (uintptr_t)c.ld % 16 || (uintptr_t)c.lt % 16) return DSPARK_ENOTIMPL;
  const SvLayout Ly = sv_layout(c.B, c.gamma, c.V);
  if (c.ws_bytes < Ly.total) return DSPARK_ENOTIMPL;
  const bool greedy = c.T == 0.f;
  const int ntile = (c.V + kSvTile - 1) / kSvTile;
  const int rows = c.B * (c.gamma + 1);
  // clusters of 3 (45 clusters on 148 SMs) stream many rows best; with fewer than about 1.3 rows
  // per cluster, clusters of 6 spread each row over more SMs (measured on a B200: 39.0 -> 32.8 us
  // at B = 1, gamma = 7; 129.1 -> 122.9 us at B = 32, gamma = 4; 341 -> 388 us at B = 64,
  // gamma = 16, where 3 stays)
  int C = opt.verify_stream_cluster;
  if (C < 1 || C > kSvMaxCluster) C = ((long long)rows * 3 < (long long)device_sm_count() * 4) ? 6 : 3;
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
  a.lt_off = c.lt_off;
  a.lt_nrows = c.lt_nrows;
  ld_strides(c.ld_layout, c.B, c.gamma, c.V, a.ld_sk, a.ld_sb);
  a.njobs = c.B * (c.gamma + 1);
  a.ntile = ntile;
  a.lag = 1;  // a row's second pass right after the next row's first (lags of 0, 2 and 3 measured slower)
  a.l2hint = opt.verify_stream_l2hint;
  a.wait_ns = opt.debug_wait_limit > 0 ? (uint64_t)std::min<long>(opt.debug_wait_limit, (long)kSvTimeoutNs) : kSvTimeoutNs;
  a.xbar_extra = opt.debug_unreachable_barrier == 2 ? 1 : 0;
  a.greedy = greedy ? 1 : 0;
  a.zscale = a.greedy ? 0.f : (float)(1.4426950408889634 / (double)c.T);
  a.do_verify = 1;
  a.c_star = c.c_star;
  a.n_acc = c.n_acc;
  a.y_out = c.y_out;
  a.flags = c.flags;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.rej = reinterpret_cast<int*>(ws + Ly.rej);
  a.rows = reinterpret_cast<SvRow*>(ws + Ly.rows);
  a.part = reinterpret_cast<double2*>(ws + Ly.part);
  a.trec = reinterpret_cast<float2*>(ws + Ly.trec);
  a.qrec = reinterpret_cast<float*>(ws + Ly.qrec);
  auto kern = a.greedy ? verify_stream<true> : verify_stream<false>;
  const size_t smem = kSvRingBytes;
  cudaError_t rc;
  rc = ensure_smem_attr((const void*)kern, smem);
  if (rc == cudaSuccess && C > 8) rc = ensure_nonportable_cluster((const void*)kern);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(verify_stream): ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  rc = cudaMemsetAsync(ws, 0, Ly.rows, c.stream);  // status word and the rejection records
  if (rc != cudaSuccess) {
    set_error(std::string("cudaMemsetAsync: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kSvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int ncl = 0;
  for (; C >= 1; --C) {  // a cluster size the device cannot hold: try smaller ones
    if (C > 8 && ensure_nonportable_cluster((const void*)kern) != cudaSuccess) {
      (void)cudaGetLastError();
      break;
    }
    attr[0].val.clusterDim.x = C;
    cfg.gridDim = dim3((unsigned)C);
    if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) == cudaSuccess && ncl > 0) break;
    (void)cudaGetLastError();
    ncl = 0;
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
