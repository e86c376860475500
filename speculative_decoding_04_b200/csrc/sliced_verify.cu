// Column-sliced verification: the rejection-sampling verify and the TV labels with every row of
// l_d and l_t read from HBM exactly once.
//
// [P1 "DeepSeek V4-Pro DSpark 推测解码方案深度解析" §大模型推理的显存瓶颈与推测解码的演进逻辑:
//  the target checks the drafted tokens left to right with rejection sampling, keeps the
//  longest passing prefix, resamples one token at the first failure and drops the rest]
// [P3 "DSpark Speculative Decoding", opening paragraph: longest consistent prefix + bonus token;
//  §Confidence-Scheduled Verification: label c*_k = 1 - ½‖p_d - p_t‖₁]
//
// Layout of the work.  The grid (one CTA per SM, all resident) is cut into G groups of P CTAs.
// A job is one position k of one request b: the draft row l_d[k,b] and the target row
// l_t[b,k].  Group g takes the jobs j = g, g + G, g + 2G, ... (position-major j = k*B + b) that
// need any row; CTA r of the group owns the r-th of P contiguous column slices of every row
// (about 4 KB of each row at V = 151936, P = 37: one 16 KB bulk copy per row and job).
// Per job each CTA
//   P1  (slice from HBM into a shared-memory stage)  per pass-1 warp a tile of the slice: the integer
//       reference R_w = ceil(max l * c) (c = log2(e)/T), the exponentials e = 2^fma(l, c, -R_w),
//       written back in place, and their sum; the CTA's (R, S) for l_d and l_t go to a record
//       in global memory;
//   --  every CTA of the group polls the job's P records until all are there, folds them in rank
//       order into the row normalisers log2 p = l c - K - lam (the same bits in every CTA) and
//       decides the acceptance from the two logits at the drafted token, in fp64;
//   P2  (the same stage, still resident)  p = e * 2^(R_w - K - lam): sum min(p_d, p_t) for the
//       label, whether any column has p_t > p_d, and for a rejected row (its residual) or the
//       bonus row per-tile sums of q = max(0, p_t - p_d) and of p_t.
// A record is eight 8-byte words, each a 4-byte payload and the call's 32-bit tag: an aligned
// 8-byte store is single-copy atomic, so a reader that sees the tag in every word has the whole
// record, and the writer needs no fence (a release fence per job, waiting for the store to
// reach L2 under the copy stream's load, serialised the exchange at about 2 us a job).
// The stage is free again after P2.  P1 and P2 run on separate warps, so the first passes of
// later jobs go on while a job waits for its group's records; the ring holds the jobs between
// their copy and their P2.  Greedy verification (T = 0) needs P1 (top-2 of each row) only.
//
// Roles in a CTA of 800 threads: warp 16 issues the bulk copies; warps 0-7 run P1 and warps 8-15
// P2, one 1/8 tile of the slice each (two sets, so that P1 never waits behind a decision); the
// last P1 warp to finish a job folds the eight partials and publishes the CTA's record; warps
// 17-24 each collect the group's records of every eighth job, decide, and hand the normalisers
// to P2.
// A small second kernel (one warp per request) finds n, samples the residual / bonus token by
// an inverse CDF over the per-tile sums and one rescanned tile, and writes y, n, c*.
// Every wait is bounded; after a timeout all roles stop and the status word is set.

#include <algorithm>
#include <atomic>
#include <cfloat>
#include <chrono>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace dspark {

namespace {

constexpr int kVsTiles = 8;                         // tiles per slice: one pass-1 and one pass-2 warp each
constexpr int kVsDeciders = 8;                      // decider warps: job i goes to decider i % 8
constexpr int kVsThreads = (2 * kVsTiles + 1 + kVsDeciders) * 32;  // + producer, deciders
constexpr int kVsProducer = 2 * kVsTiles;
constexpr int kVsDecider = 2 * kVsTiles + 1;
constexpr int kVsMaxStages = 8;
constexpr int kVsSlots = 16;                        // ring of per-job partials and decisions
constexpr int kVsMaxNQ = 8;                         // float4s per lane and row of a tile
constexpr int kVsMaxP = 160;                        // CTAs per group
constexpr int kVsMaxJobs = 8192;                    // jobs of one group (descriptors in shared memory)
constexpr int kVsSmemLimit = 227 * 1024;
constexpr uint32_t kVsSuspendNs = 100000;
constexpr uint64_t kVsTimeoutNs = 2000000000ull;    // a wait gives up after 2 s
constexpr int kRNone = -(1 << 28);                  // reference of an empty sum
constexpr int kRMax = 1 << 24;

// One CTA's pass-1 result for one job: (R, S) pairs of l_d and l_t, or greedy top-2 (the
// payload of a tagged record in global memory).
struct __align__(16) VsRec {
  union {
    struct {
      double Sd, St;
      int Rd, Rt;
    } sm;
    struct {
      Top2 gd, gt;
    } gr;
  };
  uint32_t fl;
  uint32_t pad;
};
static_assert(sizeof(VsRec) == 32, "record size");
constexpr int kVsRecWords = 8;  // 8-byte words of a tagged record: 4-byte payload | 4-byte tag
static_assert(kVsSlots % kVsDeciders == 0, "a slot's jobs must meet one decider");

// Normalisers of a job's rows and what P2 must produce.
struct __align__(16) VsDec {
  float Kd, lamd, Kt, lamt;
  int what;  // bit 0 labels, bit 1 residual sums (rejected row), bit 2 bonus sums
  int pad0, pad1, pad2;
};

// Per-job record read by the finalize kernel.
struct __align__(16) VsRow {
  float Kd, lamd, Kt, lamt;
  int acc;
  uint32_t fl;  // ACCEPT_NEAR_TIE / SAMPLE_NEAR_TIE
  int cand;     // greedy: argmax of l_t
  float cstar;  // greedy label
};

struct VsArgs {
  const float* ld;
  const float* lt;
  const int32_t* x;
  const int32_t* L;
  const float* u_acc;
  const float* u_res;
  int B, gamma, V, lt_rows;
  int G, P, NS, wmax, nq, njobs;
  size_t ld_sk, ld_sb;  // element strides of the l_d row of position k and request b
  float zc;  // log2(e) / T (T > 0)
  int greedy;
  float* c_star;
  int32_t* n_acc;
  int32_t* y_out;
  uint32_t* flags;
  uint32_t* status;
  uint32_t tag;    // this call's tag (never 0)
  unsigned long long* xrec;  // [njobs][P][8] tagged records
  VsRow* rows;     // [njobs]
  double2* part;   // [njobs][P]: (sum min(p_d, p_t), any p_t > p_d) of each CTA (k < gamma)
  float2* trec;    // [njobs][P * 8]: (sum q, sum p_t) of each tile (rejected and bonus rows)
};

struct VsJob {
  int b, k, j;
  bool d, t, verify, bonus, cstar;
};

__device__ __forceinline__ VsJob vs_job(const VsArgs& a, int j) {
  VsJob J;
  J.j = j;
  J.k = j / a.B;
  J.b = j - J.k * a.B;
  int Lb = a.gamma;
  if (a.L) Lb = min(max(__ldg(a.L + J.b), 0), a.gamma);
  J.cstar = a.c_star != nullptr && J.k < a.gamma;
  J.verify = J.k < Lb;
  J.bonus = J.k == Lb;
  J.d = J.cstar || (J.verify && !a.greedy);  // greedy acceptance needs only argmax l_t
  J.t = J.cstar || J.verify || J.bonus;
  return J;
}

// Quads [q0, q1) of slice r (P contiguous slices of the V/4 quads).
__device__ __forceinline__ int vs_q0(int r, int nq, int P) { return (int)((long long)r * nq / P); }
// Barrier over `nthreads` threads that also returns whether v holds in all of them (so that a
// group of warps leaves a loop together: none may wait at a barrier another has abandoned).
__device__ __forceinline__ bool bar_and(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float vs_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ double vs_pow2d(int d) {
  return d < -1022 ? 0.0 : (d > 1023 ? INFINITY : __longlong_as_double((long long)(1023 + d) << 52));
}
// Integer reference of a maximum m of raw logits: R = ceil(m c), clamped; kRNone for no maximum.
__device__ __forceinline__ int vs_ref(float m, float c) {
  if (!(m > -INFINITY)) return kRNone;
  const int R = __float2int_ru(m * c);
  return min(max(R, -kRMax), kRMax);
}
// Scale of a tile whose exponentials were taken against R_w: 2^(R_w - K - lam).  The same
// expression in P2 and in the finalize's rescan, so both see the same bits.
__device__ __forceinline__ float vs_scale(int Rw, float K, float lam) {
  return Rw == kRNone ? 0.f : vs_ex2(__fsub_rn(__fsub_rn((float)Rw, K), lam));
}
// Normalisers (K, lam) from (R, S): S = f 2^e with f in [0.5, 1), K = R + e - 1, lam = log2(2f).
__device__ __forceinline__ bool vs_norm(int R, double S, float& K, float& lam) {
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

__device__ __forceinline__ uint64_t vs_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool vs_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kVsSuspendNs)
      : "memory");
  return ok != 0;
}

struct VsSync {
  volatile int* abort;
  uint32_t* status;
  __device__ void give_up() const {
    *abort = 1;
    atomicOr(status, (uint32_t)DSPARK_ETIMEOUT);
  }
};

// Bounded mbarrier wait (2 s); returns false at once once any role has given up.
__device__ __forceinline__ bool vs_wait(const VsSync& s, uint64_t* bar, uint32_t parity) {
  if (*s.abort) return false;
  if (vs_try_wait(bar, parity)) return true;
  const uint64_t t0 = vs_now();
  while (true) {
    if (vs_try_wait(bar, parity)) return true;
    if (*s.abort) return false;
    if (vs_now() - t0 > kVsTimeoutNs) break;
  }
  s.give_up();
  return false;
}

// Payload word w of a record (w < 7).
__device__ __forceinline__ VsRec vs_empty_rec(bool greedy);
__device__ __forceinline__ VsRec vs_fold_lanes(VsRec r, bool greedy);
__device__ __forceinline__ void vs_fold_one(VsRec& acc, const VsRec& o, bool greedy);

__device__ __forceinline__ uint32_t vs_word(const VsRec& r, int w, bool greedy) {
  if (greedy) {
    switch (w) {
      case 0: return __float_as_uint(r.gr.gd.best);
      case 1: return (uint32_t)r.gr.gd.idx;
      case 2: return __float_as_uint(r.gr.gd.second);
      case 3: return __float_as_uint(r.gr.gt.best);
      case 4: return (uint32_t)r.gr.gt.idx;
      case 5: return __float_as_uint(r.gr.gt.second);
      default: return r.fl;
    }
  }
  switch (w) {
    case 0: return (uint32_t)r.sm.Rd;
    case 1: return (uint32_t)r.sm.Rt;
    case 2: return (uint32_t)__double2loint(r.sm.Sd);
    case 3: return (uint32_t)__double2hiint(r.sm.Sd);
    case 4: return (uint32_t)__double2loint(r.sm.St);
    case 5: return (uint32_t)__double2hiint(r.sm.St);
    default: return r.fl;
  }
}

__device__ __forceinline__ VsRec vs_unpack(const uint32_t (&w)[kVsRecWords], bool greedy) {
  VsRec r;
  if (greedy) {
    r.gr.gd = Top2{__uint_as_float(w[0]), (int)w[1], __uint_as_float(w[2])};
    r.gr.gt = Top2{__uint_as_float(w[3]), (int)w[4], __uint_as_float(w[5])};
  } else {
    r.sm.Rd = (int)w[0];
    r.sm.Rt = (int)w[1];
    r.sm.Sd = __hiloint2double((int)w[3], (int)w[2]);
    r.sm.St = __hiloint2double((int)w[5], (int)w[4]);
  }
  r.fl = w[6];
  r.pad = 0;
  return r;
}

// Lanes 0-7 store one tagged word each (no fence: every word is self-validating).
__device__ __forceinline__ void vs_publish(unsigned long long* rec, const VsRec& r, uint32_t tag, bool greedy) {
  const int lane = threadIdx.x & 31;
  if (lane < kVsRecWords) {
    const unsigned long long v = (unsigned long long)vs_word(r, lane, greedy) | ((unsigned long long)tag << 32);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(rec + lane), "l"(v) : "memory");
  }
}

// Poll (whole warp, bounded) until the P tagged records of a job are all there, then fold them:
// lane l folds records l, l + 32, ... in order, then the lanes are folded (the same bits in every
// CTA that reads the same records).
__device__ __forceinline__ bool vs_collect(const VsSync& s, const unsigned long long* recs, int P, uint32_t tag,
                                           bool greedy, VsRec& out) {
  const int lane = threadIdx.x & 31;
  uint64_t t0 = 0;
  while (true) {
    // a cheap poll first (one word of each record, with a pause between polls: eight deciders
    // per CTA polling whole records without pausing slowed the copy stream through L2)
    bool seen = true;
    for (int r = lane; r < P; r += 32) {
      unsigned long long v;
      asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(recs + (size_t)r * kVsRecWords + 6) : "memory");
      seen &= (uint32_t)(v >> 32) == tag;
    }
    if (!__all_sync(0xffffffffu, seen)) {
      if (*s.abort) return false;
      const uint64_t t = vs_now();
      if (t0 == 0) t0 = t;
      else if (t - t0 > kVsTimeoutNs) {
        if (lane == 0) s.give_up();
        __syncwarp();
        return false;
      }
      __nanosleep(256);
      continue;
    }
    VsRec acc = vs_empty_rec(greedy);
    bool all = true;
    for (int r = lane; r < P; r += 32) {
      uint32_t w[kVsRecWords];
      bool ok = true;
#pragma unroll
      for (int h = 0; h < kVsRecWords; h += 2) {
        unsigned long long a, b;
        asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];"
                     : "=l"(a), "=l"(b)
                     : "l"(recs + (size_t)r * kVsRecWords + h)
                     : "memory");
        ok &= (uint32_t)(a >> 32) == tag && (uint32_t)(b >> 32) == tag;
        w[h] = (uint32_t)a;
        w[h + 1] = (uint32_t)b;
      }
      all &= ok;
      if (ok) vs_fold_one(acc, vs_unpack(w, greedy), greedy);
    }
    if (__all_sync(0xffffffffu, all)) {
      out = vs_fold_lanes(acc, greedy);
      return true;
    }
    if (*s.abort) return false;
    const uint64_t t = vs_now();
    if (t0 == 0) t0 = t;
    else if (t - t0 > kVsTimeoutNs) {
      if (lane == 0) s.give_up();
      __syncwarp();
      return false;
    }
  }
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float vs_warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Fold of (R, S) pairs held by the lanes of a warp: every lane returns the same bits.
__device__ __forceinline__ void vs_warp_fold(int& R, double& S) {
  const int M = __reduce_max_sync(0xffffffffu, R);
  double v = (R == kRNone) ? 0.0 : S * vs_pow2d(R - M);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  R = M;
  S = v;
}

__device__ __forceinline__ Top2 vs_top2_warp(Top2 t) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = top2_merge(t, top2_shfl_xor(t, o));
  return t;
}

__device__ __forceinline__ VsRec vs_empty_rec(bool greedy) {
  VsRec r;
  if (greedy) {
    r.gr.gd = Top2{-INFINITY, -1, -INFINITY};
    r.gr.gt = Top2{-INFINITY, -1, -INFINITY};
  } else {
    r.sm.Sd = r.sm.St = 0.0;
    r.sm.Rd = r.sm.Rt = kRNone;
  }
  r.fl = 0;
  r.pad = 0;
  return r;
}

// Fold of the records of lanes 0..31 (each already holding the lane's fold of records
// lane, lane + 32, ...) into one, identical in every lane.
__device__ __forceinline__ VsRec vs_fold_lanes(VsRec r, bool greedy) {
  if (greedy) {
    r.gr.gd = vs_top2_warp(r.gr.gd);
    r.gr.gt = vs_top2_warp(r.gr.gt);
  } else {
    vs_warp_fold(r.sm.Rd, r.sm.Sd);
    vs_warp_fold(r.sm.Rt, r.sm.St);
  }
  r.fl = __reduce_or_sync(0xffffffffu, r.fl);
  return r;
}

// Sequential fold of one more record into a lane's running record (exact power-of-two rescale).
__device__ __forceinline__ void vs_fold_one(VsRec& acc, const VsRec& o, bool greedy) {
  if (greedy) {
    acc.gr.gd = top2_merge(acc.gr.gd, o.gr.gd);
    acc.gr.gt = top2_merge(acc.gr.gt, o.gr.gt);
  } else {
    auto f = [](int& R, double& S, int r, double s) {
      if (r == kRNone) return;
      if (R == kRNone) {
        R = r;
        S = s;
        return;
      }
      const int M = max(R, r);
      S = S * vs_pow2d(R - M) + s * vs_pow2d(r - M);
      R = M;
    };
    f(acc.sm.Rd, acc.sm.Sd, o.sm.Rd, o.sm.Sd);
    f(acc.sm.Rt, acc.sm.St, o.sm.Rt, o.sm.St);
  }
  acc.fl |= o.fl;
}

// Per-warp pass-1 partial in shared memory.
struct __align__(16) VsWarpPart {
  union {
    struct {
      float Sd, St;
      int Rd, Rt;
    } sm;
    struct {
      Top2 gd, gt;
    } gr;
  };
  uint32_t fl;
  uint32_t pad;
};

// Job descriptor (built once per launch): request b (bits 0-19), position k (bits 20-26) and
// what the job needs.
constexpr uint32_t kJobD = 1u << 27, kJobVerify = 1u << 28, kJobBonus = 1u << 29, kJobCstar = 1u << 30;

struct VsJd {
  int b, k, j;
  bool d, verify, bonus, cstar;
};

__device__ __forceinline__ uint32_t vs_pack(const VsJob& J) {
  return (uint32_t)J.b | ((uint32_t)J.k << 20) | (J.d ? kJobD : 0u) | (J.verify ? kJobVerify : 0u) |
         (J.bonus ? kJobBonus : 0u) | (J.cstar ? kJobCstar : 0u);
}
__device__ __forceinline__ VsJd vs_unpack_jd(uint32_t w, int B) {
  VsJd J;
  J.b = (int)(w & 0xFFFFFu);
  J.k = (int)((w >> 20) & 127u);
  J.j = J.k * B + J.b;
  J.d = (w & kJobD) != 0;
  J.verify = (w & kJobVerify) != 0;
  J.bonus = (w & kJobBonus) != 0;
  J.cstar = (w & kJobCstar) != 0;
  return J;
}

// Quads of tile w (kVsTiles per slice) relative to the slice start.
__device__ __forceinline__ int vs_t0(int w, int ns) { return w * ns / kVsTiles; }

__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 f2add(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Pass 1 over one row of a tile (lane l takes quads l, l + 32, ...): the tile's reference
// R = ceil(max l * c) over the warp, e = 2^fma(l, c, -R) written back in place, and the lane's
// fp32 sum of e.  Packed fp32 pairs round each element exactly like the scalar instructions.
template <int NQ>
__device__ __forceinline__ float vs_row_p1(float* row, int nw, float zc, int& R) {
  const int lane = threadIdx.x & 31;
  float4 v[NQ];
  float m = -INFINITY;
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int qi = lane + 32 * q;
    v[q] = qi < nw ? *reinterpret_cast<const float4*>(row + qi * 4)
                   : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    m = fmax3f(fmax3f(m, v[q].x, v[q].y), v[q].z, v[q].w);
  }
  R = __reduce_max_sync(0xffffffffu, vs_ref(m, zc));
  const float2 c2 = make_float2(zc, zc), n2 = make_float2(-(float)R, -(float)R);
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int qi = lane + 32 * q;
    const float2 x = f2fma(make_float2(v[q].x, v[q].y), c2, n2), y = f2fma(make_float2(v[q].z, v[q].w), c2, n2);
    const float4 e = make_float4(vs_ex2(x.x), vs_ex2(x.y), vs_ex2(y.x), vs_ex2(y.y));
    acc = f2add(acc, make_float2(e.x, e.y));
    acc = f2add(acc, make_float2(e.z, e.w));
    if (qi < nw) *reinterpret_cast<float4*>(row + qi * 4) = e;
  }
  return acc.x + acc.y;
}

template <bool GREEDY, int NQ>
__global__ void __launch_bounds__(kVsThreads, 1) verify_sliced(VsArgs a) {
  extern __shared__ __align__(128) uint8_t vs_smem[];
  float* ring = reinterpret_cast<float*>(vs_smem);                                      // [NS][2][wmax]
  uint32_t* jd = reinterpret_cast<uint32_t*>(vs_smem + (size_t)a.NS * 2 * a.wmax * 4);  // job descriptors
  __shared__ __align__(8) uint64_t full[kVsMaxStages], empty[kVsMaxStages];
  __shared__ __align__(8) uint64_t pbar[kVsSlots], dbar[kVsSlots];
  __shared__ int pcount[kVsSlots];  // pass-1 warps done with the slot's job
  __shared__ VsWarpPart wpart[kVsSlots][kVsTiles];
  __shared__ int2 wref[kVsSlots][kVsTiles];      // pass-1 references (l_d, l_t) of each tile
  __shared__ float2 w2part[kVsSlots][kVsTiles];  // (sum min, any p_t > p_d) of each tile
  __shared__ VsDec dec[kVsSlots];
  __shared__ int s_abort, s_njobs;
  __shared__ int s_scan[kVsThreads / 32 + 1];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x / a.P, rank = blockIdx.x - g * a.P;
  const VsSync sy{&s_abort, a.status};
  const int P = a.P, G = a.G;
  constexpr unsigned FULL = 0xffffffffu;

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kVsTiles);  // the pass-2 warps (the pass-1 warps when greedy)
    }
    for (int i = 0; i < kVsSlots; ++i) {
      mbar_init(&pbar[i], kVsTiles);
      mbar_init(&dbar[i], 1);
      pcount[i] = 0;
    }
    s_abort = 0;
    fence_mbar_init();
  }
  // ---- this group's jobs that read anything, in job order (block-wide compaction)
  {
    int base = 0;
    const int per_group = (a.njobs - g + G - 1) / G;
    for (int c0 = 0; c0 < per_group; c0 += kVsThreads) {
      const int i = c0 + (int)threadIdx.x;
      VsJob J;
      bool need = false;
      if (i < per_group) {
        J = vs_job(a, g + i * G);
        need = J.t;
      }
      const unsigned m = __ballot_sync(FULL, need);
      if (lane == 0) s_scan[warp] = __popc(m);
      __syncthreads();
      if (threadIdx.x == 0) {
        int sum = 0;
        for (int w = 0; w < kVsThreads / 32; ++w) {
          const int v = s_scan[w];
          s_scan[w] = sum;
          sum += v;
        }
        s_scan[kVsThreads / 32] = sum;
      }
      __syncthreads();
      if (need) jd[base + s_scan[warp] + __popc(m & ((1u << lane) - 1u))] = vs_pack(J);
      base += s_scan[kVsThreads / 32];
      __syncthreads();
    }
    if (threadIdx.x == 0) s_njobs = base;
    __syncthreads();
  }
  const int n = s_njobs;
  const int q0 = vs_q0(rank, a.nq, P), ns = vs_q0(rank + 1, a.nq, P) - q0;  // slice: quads [q0, q0 + ns)
  const float zc = a.zc;

  if (warp == kVsProducer) {
    // ------------------------------------------------------------------ bulk copies, one per row and job
    if (lane == 0) {
      int i = 0;
      bool ok = true;
      const uint32_t bytes = (uint32_t)ns * 16u;
      for (; i < n; ++i) {
        const int s = i % a.NS;
        if (!vs_wait(sy, &empty[s], ((i / a.NS) & 1) ^ 1)) {
          ok = false;
          break;
        }
        const VsJd J = vs_unpack_jd(jd[i], a.B);
        float* st = ring + (size_t)s * 2 * a.wmax;
        mbar_expect_tx(&full[s], bytes ? (J.d ? 2u : 1u) * bytes : 0u);
        if (bytes) {
          if (J.d) bulk_g2s(st, a.ld + (size_t)J.k * a.ld_sk + (size_t)J.b * a.ld_sb + (size_t)q0 * 4, bytes, &full[s]);
          bulk_g2s(st + a.wmax, a.lt + ((size_t)J.b * a.lt_rows + J.k) * a.V + (size_t)q0 * 4, bytes, &full[s]);
        }
        mbar_arrive(&full[s]);
      }
      if (!ok) {
        // let the copies still in flight land before the CTA can exit
        for (int ii = max(0, i - a.NS); ii < i; ++ii)
          for (uint32_t t = 0; t < kSpinLimit && !mbar_try_wait(&full[ii % a.NS], (ii / a.NS) & 1); ++t) {
          }
      }
    }
  } else if (warp < kVsTiles) {
    // ------------------------------------------------------------------ pass 1 of tile `warp` of every job
    const int w = warp;
    const int w0 = vs_t0(w, ns), nw = vs_t0(w + 1, ns) - w0;  // quads [w0, w0 + nw) of the slice
    const int vbase = (q0 + w0) * 4;                          // vocabulary index of the tile
    bool ok = true;
    for (int i = 0; ok && i < n; ++i) {
      const int s = i % a.NS, slot = i % kVsSlots;
      const VsJd J = vs_unpack_jd(jd[i], a.B);
      ok = __all_sync(FULL, vs_wait(sy, &full[s], (i / a.NS) & 1));
      if (!ok) break;
      float* sd = ring + (size_t)s * 2 * a.wmax + w0 * 4;
      float* st = sd + a.wmax;
      VsWarpPart out;
      if (GREEDY) {
        // top-2 of each row of the tile, one row at a time; then the stage is free
        bool bad = false;
        auto top2_row = [&](const float* row) {
          Top2 t{-INFINITY, -1, -INFINITY};
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const int qi = lane + 32 * q;
            if (qi < nw) {
              const float4 v = *reinterpret_cast<const float4*>(row + qi * 4);
              const float e[4] = {v.x, v.y, v.z, v.w};
              const int base = vbase + qi * 4;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                bad |= isnan(e[c]) || e[c] == INFINITY;
                if (e[c] > -INFINITY) top2_push(t, e[c], base + c);
              }
            }
          }
          return vs_top2_warp(t);
        };
        out.gr.gt = top2_row(st);
        out.gr.gd = J.d ? top2_row(sd) : Top2{-INFINITY, -1, -INFINITY};
        out.fl = __any_sync(FULL, bad) ? (uint32_t)DSPARK_FLAG_NONFINITE : 0u;
      } else {
        int Rd = kRNone, Rt = kRNone;
        float sdl = 0.f;
        if (J.d) sdl = vs_row_p1<NQ>(sd, nw, zc, Rd);
        const float stl = vs_row_p1<NQ>(st, nw, zc, Rt);
        out.sm.Sd = vs_warp_sum_f(sdl);
        out.sm.St = vs_warp_sum_f(stl);
        out.sm.Rd = Rd;
        out.sm.Rt = Rt;
        // a NaN or +Inf logit makes a sum non-finite
        out.fl = (out.sm.St <= FLT_MAX && out.sm.Sd <= FLT_MAX) ? 0u : (uint32_t)DSPARK_FLAG_NONFINITE;
        fence_proxy_async_smem();  // the exponentials (generic stores) precede the stage's next bulk copy
        if (lane == 0) wref[slot][w] = make_int2(Rd, Rt);
      }
      out.pad = 0;
      // The slot's previous job (i - 16) was read before this one can be written: its last pass-1
      // warp read it before releasing the stage's job (greedy) or before the job's decision, which
      // every stage refill since has waited for.
      int last = 0;
      if (lane == 0) {
        wpart[slot][w] = out;
        __threadfence_block();
        last = atomicAdd(&pcount[slot], 1) == kVsTiles - 1;
      }
      last = __shfl_sync(FULL, last, 0);
      if (GREEDY) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (last) {
        // the last pass-1 warp of the job folds the eight partials and publishes the CTA's record
        __threadfence_block();
        VsRec r = vs_empty_rec(GREEDY);
        if (lane < kVsTiles) {
          const VsWarpPart wp = wpart[slot][lane];
          if (GREEDY) {
            r.gr.gd = wp.gr.gd;
            r.gr.gt = wp.gr.gt;
          } else {
            r.sm.Rd = wp.sm.Rd;
            r.sm.Rt = wp.sm.Rt;
            r.sm.Sd = (double)wp.sm.Sd;
            r.sm.St = (double)wp.sm.St;
          }
          r.fl = wp.fl;
        }
        r = vs_fold_lanes(r, GREEDY);
        vs_publish(a.xrec + ((size_t)J.j * P + rank) * kVsRecWords, r, a.tag, GREEDY);
        if (lane == 0) pcount[slot] = 0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pbar[slot]);
    }
  } else if (warp < 2 * kVsTiles) {
    // ------------------------------------------------------------------ pass 2 of tile `warp - 8` (T > 0)
    if (!GREEDY) {
      const int w = warp - kVsTiles;
      const int w0 = vs_t0(w, ns), nw = vs_t0(w + 1, ns) - w0;
      bool ok = true;
      for (int i = 0; ok && i < n; ++i) {
        const int s = i % a.NS, slot = i % kVsSlots;
        // pass 1 of the job (its exponentials and references) and then its decision; a warp whose
        // wait gave up computes nothing and leaves with the others at the barrier below
        bool okw = __all_sync(FULL, vs_wait(sy, &pbar[slot], (i / kVsSlots) & 1));
        if (okw) okw = __all_sync(FULL, vs_wait(sy, &dbar[slot], (i / kVsSlots) & 1));
        VsDec dd = dec[slot];
        if (!okw) dd.what = 0;
        const VsJd J = vs_unpack_jd(jd[i], a.B);
        const float* sd = ring + (size_t)s * 2 * a.wmax + w0 * 4;
        const float* st = sd + a.wmax;
        float smin = 0.f, qs = 0.f, pts = 0.f;
        bool anyq = false;
        if (dd.what) {
          const int2 rw = wref[slot][w];
          const float ft = vs_scale(rw.y, dd.Kt, dd.lamt);
          const float2 ft2 = make_float2(ft, ft);
          float2 sm2 = make_float2(0.f, 0.f), q2 = make_float2(0.f, 0.f), t2 = make_float2(0.f, 0.f);
          float dmax = -INFINITY;
          if (dd.what & 3) {  // labels or residual sums: both rows
            const float fd = vs_scale(rw.x, dd.Kd, dd.lamd);
            const float2 fd2 = make_float2(fd, fd), mone = make_float2(-1.f, -1.f);
            const bool resid = (dd.what & 6) != 0;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              const int qi = lane + 32 * q;
              if (qi < nw) {
                const float4 ed = *reinterpret_cast<const float4*>(sd + qi * 4);
                const float4 et = *reinterpret_cast<const float4*>(st + qi * 4);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const float2 pd = f2mul(h ? make_float2(ed.z, ed.w) : make_float2(ed.x, ed.y), fd2);
                  const float2 pt = f2mul(h ? make_float2(et.z, et.w) : make_float2(et.x, et.y), ft2);
                  sm2 = f2add(sm2, make_float2(fminf(pd.x, pt.x), fminf(pd.y, pt.y)));
                  const float2 df = f2fma(pd, mone, pt);  // p_t - p_d, rounded once
                  dmax = fmax3f(dmax, df.x, df.y);
                  if (resid) {
                    q2 = f2add(q2, make_float2(fmaxf(df.x, 0.f), fmaxf(df.y, 0.f)));
                    t2 = f2add(t2, pt);
                  }
                }
              }
            }
          } else {  // bonus sums only (l_d was not loaded)
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              const int qi = lane + 32 * q;
              if (qi < nw) {
                const float4 et = *reinterpret_cast<const float4*>(st + qi * 4);
                t2 = f2add(t2, f2mul(make_float2(et.x, et.y), ft2));
                t2 = f2add(t2, f2mul(make_float2(et.z, et.w), ft2));
              }
            }
          }
          smin = vs_warp_sum_f(sm2.x + sm2.y);
          anyq = __any_sync(FULL, dmax > 0.f);
          if (dd.what & 6) {
            qs = vs_warp_sum_f(q2.x + q2.y);
            pts = vs_warp_sum_f(t2.x + t2.y);
            if (lane == 0) a.trec[(size_t)J.j * (P * kVsTiles) + rank * kVsTiles + w] = make_float2(qs, pts);
          }
        }
        if (lane == 0) w2part[slot][w] = make_float2(smin, anyq ? 1.f : 0.f);
        // the label partial of the CTA: the first pass-2 warp folds the eight tiles' partials
        ok = bar_and(1, kVsTiles * 32, okw);
        if (!ok) break;
        if (w == 0 && J.cstar) {
          const float2 v = lane < kVsTiles ? w2part[slot][lane] : make_float2(0.f, 0.f);
          const double sm = warp_sum_d((double)v.x), nq = warp_sum_d((double)v.y);
          if (lane == 0) a.part[(size_t)J.j * P + rank] = make_double2(sm, nq);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
  } else if (warp >= kVsDecider) {
    // ------------------------------------------------------------------ fold the group's records, decide
    // Each decider takes every kVsDeciders-th job (so the jobs of one slot always meet the same
    // decider, which keeps the slot's barrier phases in order); a decision is a chain of
    // dependent global-memory round trips, and several chains run at once.
    bool ok = true;
    for (int i = warp - kVsDecider; ok && i < n; i += kVsDeciders) {
      const int slot = i % kVsSlots;
      const VsJd J = vs_unpack_jd(jd[i], a.B);
      // the drafted token, its uniform and (T > 0) the two logits at it are requested before the wait
      const int xk = J.verify ? __ldg(a.x + (size_t)J.b * a.gamma + J.k) : -1;
      const float u_acc = (J.verify && !GREEDY) ? __ldg(a.u_acc + (size_t)J.b * a.gamma + J.k) : 0.f;
      float ldx = 0.f, ltx = 0.f;
      if (!GREEDY && J.verify && (unsigned)xk < (unsigned)a.V) {
        ldx = __ldg(a.ld + (size_t)J.k * a.ld_sk + (size_t)J.b * a.ld_sb + xk);
        ltx = __ldg(a.lt + ((size_t)J.b * a.lt_rows + J.k) * a.V + xk);
      }
      VsRec x;
      ok = vs_collect(sy, a.xrec + (size_t)J.j * P * kVsRecWords, P, a.tag, GREEDY, x);
      if (!ok) break;
      VsRow row;
      row.Kd = row.lamd = row.Kt = row.lamt = 0.f;
      row.acc = 0;
      row.fl = 0;
      row.cand = 0;
      row.cstar = 0.f;
      uint32_t dfl = x.fl;
      if (GREEDY) {
        const Top2 gt = x.gr.gt, gd = x.gr.gd;
        const bool ttie = gt.best - gt.second <= 1e-6f * fmaxf(1.f, fabsf(gt.best));
        row.cand = min(max(gt.idx, 0), a.V - 1);
        if (gt.idx < 0) dfl |= DSPARK_FLAG_NONFINITE;
        row.cstar = (gd.idx == gt.idx) ? 1.f : 0.f;
        row.fl = ttie ? (DSPARK_FLAG_ACCEPT_NEAR_TIE | DSPARK_FLAG_SAMPLE_NEAR_TIE) : 0u;
        if (J.verify) {
          if ((unsigned)xk >= (unsigned)a.V) dfl |= DSPARK_FLAG_TOKEN_RANGE;
          row.acc = (xk == gt.idx) ? 1 : 0;
        }
      } else {
        bool good = vs_norm(x.sm.Rt, x.sm.St, row.Kt, row.lamt);
        if (J.d) good &= vs_norm(x.sm.Rd, x.sm.Sd, row.Kd, row.lamd);
        if (!good) dfl |= DSPARK_FLAG_NONFINITE;
        if (J.verify) {
          if ((unsigned)xk >= (unsigned)a.V) {
            dfl |= DSPARK_FLAG_TOKEN_RANGE;
          } else {
            // u p_d(x) < p_t(x) with p = 2^(l c - R) / S, in fp64 (l c is exact there)
            const double pd = exp2((double)ldx * (double)zc - (double)x.sm.Rd) / x.sm.Sd;
            const double pt = exp2((double)ltx * (double)zc - (double)x.sm.Rt) / x.sm.St;
            const double u = (double)u_acc;
            row.acc = (u * pd < pt) ? 1 : 0;
            if (pd > 0.0 && fabs(u - pt / pd) < 1e-6) row.fl |= DSPARK_FLAG_ACCEPT_NEAR_TIE;
          }
        }
        const int what = (J.cstar ? 1 : 0) | ((J.verify && !row.acc) ? 2 : 0) | (J.bonus ? 4 : 0);
        if (lane == 0) dec[slot] = VsDec{row.Kd, row.lamd, row.Kt, row.lamt, what, 0, 0, 0};
        __syncwarp();
        if (lane == 0) mbar_arrive(&dbar[slot]);  // pass 2 of this job may start
      }
      if (rank == 0 && lane == 0) {
        a.rows[J.j] = row;
        if (dfl && a.flags) atomicOr(a.flags + J.b, dfl);
      }
    }
  }
  __syncthreads();
}

// Inverse-CDF sample of job row (k, b) (one warp): weights q = max(0, p_t - p_d) when `resid`
// (falling back to p_t when their sum is 0), else p_t.  Tile sums come from the main kernel;
// the tile holding u * W is rescanned element by element with the main kernel's arithmetic
// (its reference recomputed from its own maximum, as P1 took it).
__device__ int vs_sample(const VsArgs& a, int b, int k, bool resid, const VsRow& nm, uint32_t& fl) {
  const int lane = threadIdx.x & 31;
  const int j = k * a.B + b;
  const int P = a.P, ntile = P * kVsTiles;
  const float2* tr = a.trec + (size_t)j * ntile;
  const float zc = a.zc;
  const int per = (ntile + 31) / 32;
  const int t_lo = min(lane * per, ntile), t_hi = min(t_lo + per, ntile);
  auto tile_w = [&](int t, bool use_q) -> double {
    const float2 v = __ldcg(tr + t);
    return (double)(use_q ? v.x : v.y);
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
  const unsigned m = __ballot_sync(0xffffffffu, incl > target);
  int c = 0;
  double Pbase = 0.0;
  {
    int ln;
    bool last = false;
    if (m) {
      ln = __ffs(m) - 1;
    } else {  // u * W at or above the total through rounding: the last tile with weight
      last = true;
      const unsigned pos = __ballot_sync(0xffffffffu, own > 0.0);
      ln = pos ? 31 - __clz(pos) : 0;
    }
    if (lane == ln) {
      double accw = incl - own;
      int pick = -1;
      double pick_P = accw;
      for (int t = t_lo; t < t_hi; ++t) {
        const double w = tile_w(t, resid);
        if (w > 0.0) {
          pick = t;
          pick_P = accw;
          if (!last && accw + w > target) break;
        }
        accw += w;
      }
      c = pick >= 0 ? pick : max(t_lo, 0);
      Pbase = pick_P;
    }
    c = __shfl_sync(0xffffffffu, c, ln);
    Pbase = __shfl_sync(0xffffffffu, Pbase, ln);
  }
  c = min(max(c, 0), ntile - 1);
  // ---- the tile: slice r = c / 8, tile w = c % 8
  const int r = c / kVsTiles, w = c - r * kVsTiles;
  const int q0 = vs_q0(r, a.nq, P), ns = vs_q0(r + 1, a.nq, P) - q0;
  const int v0 = (q0 + vs_t0(w, ns)) * 4, cnt = (vs_t0(w + 1, ns) - vs_t0(w, ns)) * 4;
  const float* rowd = a.ld + (size_t)k * a.ld_sk + (size_t)b * a.ld_sb + v0;
  const float* rowt = a.lt + ((size_t)b * a.lt_rows + k) * a.V + v0;
  float md = -INFINITY, mt = -INFINITY;
  for (int e = lane; e < cnt; e += 32) {
    if (resid) md = fmaxf(md, rowd[e]);
    mt = fmaxf(mt, rowt[e]);
  }
  const int Rd = __reduce_max_sync(0xffffffffu, vs_ref(md, zc));
  const int Rt = __reduce_max_sync(0xffffffffu, vs_ref(mt, zc));
  const float fd = vs_scale(Rd, nm.Kd, nm.lamd), ft = vs_scale(Rt, nm.Kt, nm.lamt);
  auto weight = [&](int e) -> float {
    const float pt = __fmul_rn(vs_ex2(fmaf(rowt[e], zc, -(float)Rt)), ft);
    if (!resid) return pt;
    const float pd = __fmul_rn(vs_ex2(fmaf(rowd[e], zc, -(float)Rd)), fd);
    return fmaxf(__fsub_rn(pt, pd), 0.f);
  };
  int tok = -1, lastv = -1;
  double lower = 0.0, upper = 0.0, run = Pbase;
  for (int e0 = 0; e0 < cnt && tok < 0; e0 += 32) {
    const int e = e0 + lane;
    const float wv = e < cnt ? weight(e) : 0.f;
    const double inc = warp_incl_scan_d((double)wv);
    const unsigned hit = __ballot_sync(0xffffffffu, wv > 0.f && run + inc > target);
    const unsigned pos = __ballot_sync(0xffffffffu, wv > 0.f);
    if (hit) {
      const int ln = __ffs(hit) - 1;
      tok = v0 + e0 + ln;
      lower = run + __shfl_sync(0xffffffffu, inc - (double)wv, ln);
      upper = run + __shfl_sync(0xffffffffu, inc, ln);
    } else if (pos) {
      lastv = v0 + e0 + 31 - __clz(pos);
    }
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (tok < 0) {  // rounding left the target past the tile: its last element with weight
    tok = lastv >= 0 ? lastv : v0;
    lower = upper = target;
  }
  if (target - lower < 1e-6 * W || upper - target < 1e-6 * W) fl |= DSPARK_FLAG_SAMPLE_NEAR_TIE;
  return min(max(tok, 0), a.V - 1);
}

// n, y, c* and flags of every request (one warp per request).
__global__ void __launch_bounds__(128) verify_sliced_finalize(VsArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * 4 + warp;
  if (b >= a.B) return;
  const int G = a.gamma, R = G + 1, B = a.B;
  const int Lb = a.L ? min(max(__ldg(a.L + b), 0), G) : G;
  const bool timed_out = __ldcg(a.status) != 0u;
  if (a.c_star) {
    for (int k = lane; k < G; k += 32) {
      const int j = k * B + b;
      float cs;
      if (a.greedy) {
        cs = a.rows[j].cstar;
      } else {
        // sum min(p_d, p_t); exactly 1 when no column has p_t > p_d (then q = 0 everywhere)
        double sm = 0.0, nq = 0.0;
        for (int r = 0; r < a.P; ++r) {
          const double2 v = a.part[(size_t)j * a.P + r];
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
    const unsigned m = __ballot_sync(0xffffffffu, k < Lb && !a.rows[k * B + b].acc);
    if (m) {
      n = k0 + __ffs(m) - 1;
      break;
    }
  }
  uint32_t fl = 0;
  for (int k = lane; k <= n && k < Lb; k += 32) fl |= a.rows[k * B + b].fl & DSPARK_FLAG_ACCEPT_NEAR_TIE;
  fl = __reduce_or_sync(0xffffffffu, fl);
  const VsRow rn = a.rows[n * B + b];
  int tok;
  if (a.greedy) {
    tok = rn.cand;
    fl |= rn.fl & DSPARK_FLAG_SAMPLE_NEAR_TIE;
  } else {
    tok = vs_sample(a, b, n, n < Lb, rn, fl);
  }
  if (timed_out) fl |= DSPARK_FLAG_DEVICE_TIMEOUT;
  int32_t* y = a.y_out + (size_t)b * R;
  for (int jj = lane; jj < R; jj += 32) y[jj] = jj < n ? a.x[(size_t)b * G + jj] : (jj == n ? tok : -1);
  if (lane == 0) {
    a.n_acc[b] = n;
    if (fl && a.flags) atomicOr(a.flags + b, fl);
  }
}

// ============================================================================ host side

struct VsLayout {
  size_t rows, xrec, part, trec, total;
};

VsLayout vs_layout(int B, int gamma, int P) {
  const size_t nj = (size_t)B * (gamma + 1);
  VsLayout L;
  L.rows = kWsHeader;
  L.xrec = L.rows + align_up(nj * sizeof(VsRow), 256);
  L.part = L.xrec + align_up(nj * P * kVsRecWords * 8, 256);
  L.trec = L.part + align_up(nj * P * sizeof(double2), 256);
  L.total = L.trec + align_up(nj * P * kVsTiles * sizeof(float2), 256);
  return L;
}

struct VsGeometry {
  int G, P, NQ, wmax, per_group;
};

// Groups of P CTAs on the device's SMs, slices of about 16 KB per row, at most 4 float4s per
// lane and row (a slice of at most 2048 quads).
VsGeometry vs_geometry(int B, int gamma, int V, int sms, int force_groups) {
  VsGeometry g{};
  const int nq = V / 4, njobs = B * (gamma + 1);
  int G = force_groups > 0 ? force_groups : (int)std::lround((double)sms * 16384.0 / ((double)V * 4.0));
  G = std::max(1, std::min(G, std::min(sms, njobs)));
  int P = sms / G;
  const int p_min = (nq + kVsTiles * 32 * kVsMaxNQ - 1) / (kVsTiles * 32 * kVsMaxNQ);
  while (P < p_min && G > 1) P = sms / --G;
  P = std::min(std::min(P, kVsMaxP), std::max(1, nq));
  g.G = G;
  g.P = P;
  const int ns_max = (nq + P - 1) / P;
  const int per_warp = (ns_max + kVsTiles - 1) / kVsTiles;
  g.NQ = (per_warp + 31) / 32;
  g.wmax = ns_max * 4;
  g.per_group = (njobs + G - 1) / G;
  return g;
}

// Tag of a call: a process-wide counter started from the clock, never 0, so that records left in
// a workspace by an earlier call (or by anything else) are not taken for this call's.
uint32_t next_tag() {
  static std::atomic<uint32_t> ctr{(uint32_t)std::chrono::steady_clock::now().time_since_epoch().count() | 1u};
  uint32_t t = ctr.fetch_add(1u);
  if (t == 0) t = ctr.fetch_add(1u);
  return t;
}

template <bool GR>
const void* vs_kernel(int NQ) {
  switch (NQ) {
    case 1: return (const void*)verify_sliced<GR, 1>;
    case 2: return (const void*)verify_sliced<GR, 2>;
    case 3: return (const void*)verify_sliced<GR, 3>;
    case 4: return (const void*)verify_sliced<GR, 4>;
    case 5: return (const void*)verify_sliced<GR, 5>;
    case 6: return (const void*)verify_sliced<GR, 6>;
    default: return (const void*)verify_sliced<GR, 8>;
  }
}

}  // namespace

// Sized for the largest group the device allows (one group of every SM), so the size does not
// depend on the group setting.
size_t sliced_verify_workspace_bytes(int B, int gamma, int V) {
  return vs_layout(B, gamma, std::min(std::min(device_sm_count(), kVsMaxP), std::max(1, V / 4))).total;
}

// DSPARK_ENOTIMPL: this call is not for the sliced kernels (V not a multiple of 4, unaligned rows,
// too small a workspace, a slice or job list that does not fit, or the grid cannot be co-resident).
dspark_status launch_verify_sliced(const VerifyCall& c) {
  const Options opt = options();
  if (!c.do_verify || c.per_row_only || opt.verify_impl != 1) return DSPARK_ENOTIMPL;
  if (c.V % 4 || (uintptr_t)c.ld % 16 || (uintptr_t)c.lt % 16) return DSPARK_ENOTIMPL;
  if (c.lt_off) return DSPARK_ENOTIMPL;  // the flattened block runs the per-row kernels
  const int sms = device_sm_count();
  const VsGeometry geo = vs_geometry(c.B, c.gamma, c.V, sms, opt.verify_groups);
  // descriptors hold b in 20 bits and k in 7
  if (geo.NQ > kVsMaxNQ || geo.per_group > kVsMaxJobs || c.B >= (1 << 20)) return DSPARK_ENOTIMPL;
  const VsLayout Ly = vs_layout(c.B, c.gamma, geo.P);
  if (c.ws_bytes < Ly.total) return DSPARK_ENOTIMPL;
  const bool greedy = c.T == 0.f;
  const void* kern = greedy ? vs_kernel<true>(geo.NQ) : vs_kernel<false>(geo.NQ);
  cudaFuncAttributes fa;
  cudaError_t rc = cudaFuncGetAttributes(&fa, kern);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaFuncGetAttributes(verify_sliced): ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  const size_t stage = (size_t)2 * geo.wmax * 4;
  const size_t jl = align_up((size_t)geo.per_group * 4, 16);  // job descriptors
  const long long room = (long long)kVsSmemLimit - (long long)fa.sharedSizeBytes - (long long)jl - 1024;
  int NS = room > 0 ? (int)std::min<long long>(kVsMaxStages, room / (long long)stage) : 0;
  if (NS < 3) return DSPARK_ENOTIMPL;
  const size_t dyn = (size_t)NS * stage + jl;
  rc = ensure_smem_attr(kern, dyn);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(verify_sliced): ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  uint8_t* ws = static_cast<uint8_t*>(c.ws);
  VsArgs a{};
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
  ld_strides(c.ld_layout, c.B, c.gamma, c.V, a.ld_sk, a.ld_sb);
  a.G = geo.G;
  a.P = geo.P;
  a.NS = NS;
  a.wmax = geo.wmax;
  a.nq = c.V / 4;
  a.njobs = c.B * (c.gamma + 1);
  a.greedy = greedy ? 1 : 0;
  a.zc = greedy ? 0.f : (float)(1.4426950408889634 / (double)c.T);
  a.c_star = c.c_star;
  a.n_acc = c.n_acc;
  a.y_out = c.y_out;
  a.flags = c.flags;
  a.status = reinterpret_cast<uint32_t*>(ws);
  a.tag = next_tag();
  a.rows = reinterpret_cast<VsRow*>(ws + Ly.rows);
  a.xrec = reinterpret_cast<unsigned long long*>(ws + Ly.xrec);
  a.part = reinterpret_cast<double2*>(ws + Ly.part);
  a.trec = reinterpret_cast<float2*>(ws + Ly.trec);
  rc = cudaMemsetAsync(ws, 0, kWsHeader, c.stream);  // status word
  if (rc != cudaSuccess) {
    set_error(std::string("cudaMemsetAsync: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(geo.G * geo.P));
  cfg.blockDim = dim3(kVsThreads);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the CTAs of a group wait on each other
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&a};
  rc = cudaLaunchKernelExC(&cfg, kern, args);
  if (rc != cudaSuccess) {
    (void)cudaGetLastError();
    return DSPARK_ENOTIMPL;  // not co-resident: another kernel takes the call
  }
  verify_sliced_finalize<<<(c.B + 3) / 4, 128, 0, c.stream>>>(a);
  rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("verify_sliced finalize launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

}  // namespace dspark
