// Fused rejection-sampling verification and TV confidence labels.
//
// [P1 "DeepSeek V4-Pro DSpark 推测解码方案深度解析" §大模型推理的显存瓶颈与推测解码的演进逻辑:
//  the target checks the drafted tokens left to right with rejection sampling, keeps the
//  longest passing prefix, resamples one token at the first failure and drops the rest]
// [P3 "DSpark Speculative Decoding", opening paragraph: longest consistent prefix + bonus token;
//  §Confidence-Scheduled Verification: label c*_k = 1 - ½‖p_d - p_t‖₁]
//
// One thread-block cluster per (request, block position) row.  The CS CTAs of a cluster
// split the vocabulary; each holds its slice of the draft row and of the target row in
// shared memory (one bulk copy each), so both tensors are read from HBM exactly once.
// Partial statistics cross the cluster through distributed shared memory:
//   A  max of z = l / T (or greedy top-2)            -> cluster max
//   B  e = exp(z - max) in place, sums               -> normalisers S_d, S_t, e at x_k
//   C  p = e / S, sum min(p_d, p_t), sum max(0, p_t - p_d)  -> c*, residual mass Z
//   D  the CTA whose slice holds u_res * W (W = Z for a residual row, S_t for the bonus
//      row) finds the token by an fp64 segment scan of its slice.
// Every row that may be the first rejection samples its residual speculatively; the last
// row of a request to finish (atomic counter) assembles n and y.

#include <cooperative_groups.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace dspark {

struct VerifyArgs {
  const float* ld;
  const float* lt;
  const int32_t* x;
  const int32_t* L;
  const float* u_acc;
  const float* u_res;
  int B, gamma, V, lt_rows, rows_per_req;
  size_t ld_sk, ld_sb;  // element strides of the l_d row of position k and request b
  const int64_t* lt_off;  // flattened l_t: request b's rows start at row lt_off[b] (null: padded)
  long long lt_nrows;
  float inv_T;
  int greedy;
  int do_verify;
  float* c_star;
  int32_t* n_acc;
  int32_t* y_out;
  uint32_t* flags;
  uint32_t* status;
  int32_t* row_acc;
  int32_t* row_cand;
  uint32_t* row_fl;
  int32_t* counter;
  int Vc;
  int bulk;
};

struct __align__(16) Slot {
  float md, mt;
  Top2 gd, gt;
  double sd, st;
  float ed_x, et_x;
  int has_x;
  int pad0;
  double smin, sq;
  int cand;
  uint32_t cand_fl;
  uint32_t data_fl;
  int pad1;
};

constexpr int kMaxWarps = 16;

// A logit that breaks the softmax: NaN or +Inf (-Inf is a masked token with probability 0).
__device__ __forceinline__ bool bad_logit(float x) { return isnan(x) || x == INFINITY; }

// exp(z - m) as 2^((z - m) log2 e); z and m are already-rounded fp32 values
__device__ __forceinline__ float vex(float z, float m) { return exp2f(__fmul_rn(__fsub_rn(z, m), kLog2e)); }

__device__ float block_max(float v, float* sh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  v = warp_max(v);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float r = sh[0];
  for (int w = 1; w < nw; ++w) r = fmaxf(r, sh[w]);
  __syncthreads();
  return r;
}

__device__ float2 block_max2(float2 v, float2* sh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  v.x = warp_max(v.x);
  v.y = warp_max(v.y);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float2 r = sh[0];
  for (int w = 1; w < nw; ++w) {
    r.x = fmaxf(r.x, sh[w].x);
    r.y = fmaxf(r.y, sh[w].y);
  }
  __syncthreads();
  return r;
}

__device__ double2 block_sum2(double a, double b, double2* sh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  a = warp_sum_d(a);
  b = warp_sum_d(b);
  if (lane == 0) sh[warp] = make_double2(a, b);
  __syncthreads();
  double2 r = sh[0];
  for (int w = 1; w < nw; ++w) {
    r.x += sh[w].x;
    r.y += sh[w].y;
  }
  __syncthreads();
  return r;
}

__device__ Top2 block_top2(Top2 t, Top2* sh) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t = top2_merge(t, top2_shfl_xor(t, o));
  if (lane == 0) sh[warp] = t;
  __syncthreads();
  Top2 r = sh[0];
  for (int w = 1; w < nw; ++w) r = top2_merge(r, sh[w]);
  __syncthreads();
  return r;
}

// Assemble n_acc / y for every request from the per-row results (one thread per request),
// after the row kernel has finished.
__global__ void verify_finalize(VerifyArgs a) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= a.B) return;
  const int Lb = a.L ? min(max(a.L[b], 0), a.gamma) : a.gamma;
  const int R = a.gamma + 1;
  const int32_t* acc = a.row_acc + (size_t)b * R;
  const uint32_t* rfl = a.row_fl + (size_t)b * R;
  int n = 0;
  while (n < Lb && acc[n]) ++n;
  uint32_t fl = 0;
  for (int j = 0; j <= n && j < Lb; ++j) fl |= rfl[j] & DSPARK_FLAG_ACCEPT_NEAR_TIE;
  fl |= rfl[n] & (DSPARK_FLAG_SAMPLE_NEAR_TIE | DSPARK_FLAG_SMALL_RESIDUAL);
  int32_t* y = a.y_out + (size_t)b * R;
  const int cand = a.row_cand[(size_t)b * R + n];
  for (int j = 0; j < R; ++j) y[j] = (j < n) ? a.x[(size_t)b * a.gamma + j] : (j == n ? cand : -1);
  a.n_acc[b] = n;
  if (a.lt_off) {
    if (ragged_mismatch(a.lt_off, a.lt_nrows, b, Lb)) fl |= DSPARK_FLAG_RAGGED_OFFSETS;
    if (a.c_star)  // no target row in the flattened block: NaN
      for (int k = Lb + 1; k < a.gamma; ++k) a.c_star[(size_t)b * a.gamma + k] = __int_as_float(0x7fc00000);
  }
  if (fl && a.flags) atomicOr(a.flags + b, fl);
}

__global__ void __launch_bounds__(512) verify_rows(VerifyArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / CS;
  const int b = row / a.rows_per_req, kk = row - b * a.rows_per_req;
  const int tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31;

  extern __shared__ __align__(16) float vsm[];
  float* sd = vsm;
  float* st = vsm + a.Vc;
  __shared__ Slot slot;
  __shared__ __align__(8) uint64_t bar;
  __shared__ double2 sh_d[kMaxWarps];
  __shared__ Top2 sh_t[kMaxWarps];
  __shared__ double sh_w[kMaxWarps];
  __shared__ float2 sh_f2[kMaxWarps];
  __shared__ double sh_wt[16], sh_wq[16];
  __shared__ double s_St, s_ft, s_pdx, s_ptx, s_Smin, s_Z;
  __shared__ float s_cd, s_ct;
  __shared__ int s_xfound;
  __shared__ uint32_t s_dfl;
  __shared__ int s_pick;
  __shared__ double s_lo, s_hi;

  int Lb = a.gamma;
  if (a.do_verify && a.L) Lb = min(max(a.L[b], 0), a.gamma);
  // a flattened l_t holds rows 0..L_b of a request only: labels exist there
  const bool need_cstar = (a.c_star != nullptr) && kk < a.gamma && (!a.lt_off || kk <= Lb);
  const bool need_acc = a.do_verify && kk < Lb;
  const bool need_bonus = a.do_verify && kk == Lb;
  const bool need_d = need_cstar || need_acc;
  const bool need_t = need_d || need_bonus;

  if (!need_t) return;  // uniform over the cluster: nothing of this row is needed

  const int v_beg = rank * a.Vc;
  const int n = max(0, min(a.V, v_beg + a.Vc) - v_beg);
  const size_t rowd = (size_t)kk * a.ld_sk + (size_t)b * a.ld_sb + v_beg;
  const size_t rowt = lt_row_index(a.lt_off, a.lt_nrows, a.lt_rows, b, kk) * a.V + v_beg;
  bool timed_out = false;

  if (tid == 0) {
    slot.cand = -1;
    slot.cand_fl = 0;
    slot.data_fl = 0;
    slot.has_x = 0;
  }
  // ------------------------------------------------------------------ load the slices
  if (a.bulk) {
    if (tid == 0) {
      mbar_init(&bar, 1);
      fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0 && n > 0) {
      const uint32_t bytes = (uint32_t)n * 4u;
      mbar_arrive_expect_tx(&bar, need_d ? 2u * bytes : bytes);
      if (need_d) bulk_g2s(sd, a.ld + rowd, bytes, &bar);
      bulk_g2s(st, a.lt + rowt, bytes, &bar);
    }
    if (n > 0) timed_out = !mbar_wait(&bar, 0);
  } else {
    for (int i = tid; i < n; i += nthr) {
      sd[i] = need_d ? a.ld[rowd + i] : 0.f;
      st[i] = a.lt[rowt + i];
    }
    __syncthreads();
  }
  if (timed_out && a.status) atomicOr(a.status, (uint32_t)DSPARK_ETIMEOUT);

  // ------------------------------------------------------------------ phase A: maxima
  const float inv_T = a.inv_T;
  const int n4 = n >> 2;
  bool nonfin = false;
  if (a.greedy) {
    Top2 gd{-INFINITY, -1, -INFINITY}, gt{-INFINITY, -1, -INFINITY};
    for (int i = tid; i < n; i += nthr) {
      const float lt_ = st[i];
      nonfin |= isnan(lt_) || lt_ == INFINITY;
      top2_push(gt, lt_, v_beg + i);
      if (need_d) {
        const float ld_ = sd[i];
        nonfin |= isnan(ld_) || ld_ == INFINITY;
        top2_push(gd, ld_, v_beg + i);
      }
    }
    gd = block_top2(gd, sh_t);
    gt = block_top2(gt, sh_t);
    if (nonfin) atomicOr(&slot.data_fl, DSPARK_FLAG_NONFINITE);
    if (tid == 0) {
      slot.gd = gd;
      slot.gt = gt;
    }
    cluster.sync();
    if (rank == 0 && tid == 0) {
      Top2 GD{-INFINITY, -1, -INFINITY}, GT{-INFINITY, -1, -INFINITY};
      uint32_t dfl = 0;
      for (int r = 0; r < CS; ++r) {
        const Slot* p = cluster.map_shared_rank(&slot, r);
        GD = top2_merge(GD, p->gd);
        GT = top2_merge(GT, p->gt);
        dfl |= p->data_fl;
      }
      const int argt = min(max(GT.idx, 0), a.V - 1);
      const bool ttie = GT.best - GT.second <= 1e-6f * fmaxf(1.f, fabsf(GT.best));
      if (need_cstar) a.c_star[(size_t)b * a.gamma + kk] = (GD.idx == GT.idx) ? 1.f : 0.f;
      const size_t ri = (size_t)b * (a.gamma + 1) + kk;
      if (need_acc) {
        const int xk = a.x[(size_t)b * a.gamma + kk];
        if ((unsigned)xk >= (unsigned)a.V) dfl |= DSPARK_FLAG_TOKEN_RANGE;
        a.row_acc[ri] = (xk == GT.idx) ? 1 : 0;
      }
      if (need_acc || need_bonus) {
        a.row_cand[ri] = argt;
        a.row_fl[ri] = ttie ? (DSPARK_FLAG_ACCEPT_NEAR_TIE | DSPARK_FLAG_SAMPLE_NEAR_TIE) : 0u;
      }
      if (timed_out) dfl |= DSPARK_FLAG_DEVICE_TIMEOUT;
      if (dfl && a.flags) atomicOr(a.flags + b, dfl);
    }
    cluster.sync();
    return;
  }

  // ------------------------------------------------------------------ pass 1: CTA maxima of z = l * (1/T)
  float md = -INFINITY, mt = -INFINITY;
  {
    const float4* sd4 = reinterpret_cast<const float4*>(sd);
    const float4* st4 = reinterpret_cast<const float4*>(st);
    for (int i = tid; i < n4; i += nthr) {
      const float4 t4 = st4[i];
      nonfin |= bad_logit(t4.x) || bad_logit(t4.y) || bad_logit(t4.z) || bad_logit(t4.w);
      mt = fmaxf(mt, fmaxf(fmaxf(__fmul_rn(t4.x, inv_T), __fmul_rn(t4.y, inv_T)),
                           fmaxf(__fmul_rn(t4.z, inv_T), __fmul_rn(t4.w, inv_T))));
      if (need_d) {
        const float4 d4 = sd4[i];
        nonfin |= bad_logit(d4.x) || bad_logit(d4.y) || bad_logit(d4.z) || bad_logit(d4.w);
        md = fmaxf(md, fmaxf(fmaxf(__fmul_rn(d4.x, inv_T), __fmul_rn(d4.y, inv_T)),
                             fmaxf(__fmul_rn(d4.z, inv_T), __fmul_rn(d4.w, inv_T))));
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += nthr) {
      nonfin |= bad_logit(st[i]);
      mt = fmaxf(mt, __fmul_rn(st[i], inv_T));
      if (need_d) {
        nonfin |= bad_logit(sd[i]);
        md = fmaxf(md, __fmul_rn(sd[i], inv_T));
      }
    }
  }
  if (nonfin) atomicOr(&slot.data_fl, DSPARK_FLAG_NONFINITE);
  {
    const float2 m2 = block_max2(make_float2(md, mt), sh_f2);
    md = m2.x;
    mt = m2.y;
  }

  // ------------------------------------------------------------------ pass 2: e = exp(z - m_cta) in place, CTA sums
  {
    float4* sd4 = reinterpret_cast<float4*>(sd);
    float4* st4 = reinterpret_cast<float4*>(st);
    float ad = 0.f, at = 0.f;
    for (int i = tid; i < n4; i += nthr) {
      float4 t4 = st4[i];
      t4.x = vex(__fmul_rn(t4.x, inv_T), mt);
      t4.y = vex(__fmul_rn(t4.y, inv_T), mt);
      t4.z = vex(__fmul_rn(t4.z, inv_T), mt);
      t4.w = vex(__fmul_rn(t4.w, inv_T), mt);
      st4[i] = t4;
      at += (t4.x + t4.y) + (t4.z + t4.w);
      if (need_d) {
        float4 d4 = sd4[i];
        d4.x = vex(__fmul_rn(d4.x, inv_T), md);
        d4.y = vex(__fmul_rn(d4.y, inv_T), md);
        d4.z = vex(__fmul_rn(d4.z, inv_T), md);
        d4.w = vex(__fmul_rn(d4.w, inv_T), md);
        sd4[i] = d4;
        ad += (d4.x + d4.y) + (d4.z + d4.w);
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += nthr) {
      st[i] = vex(__fmul_rn(st[i], inv_T), mt);
      at += st[i];
      if (need_d) {
        sd[i] = vex(__fmul_rn(sd[i], inv_T), md);
        ad += sd[i];
      }
    }
    const double2 s2 = block_sum2((double)ad, (double)at, sh_d);
    if (tid == 0) {
      slot.md = md;
      slot.mt = mt;
      slot.sd = s2.x;
      slot.st = s2.y;
      if (need_acc) {
        const int xk = a.x[(size_t)b * a.gamma + kk];
        if (xk >= v_beg && xk < v_beg + n) {
          slot.ed_x = sd[xk - v_beg];
          slot.et_x = st[xk - v_beg];
          slot.has_x = 1;
        }
      }
    }
  }
  cluster.sync();  // (1) every CTA's (max, sum) pair is visible

  // warp 0 combines the CS pairs: lane r reads rank r; totals in rank order via a fixed scan
  if (warp == 0) {
    const bool live = lane < CS;
    const Slot* p = cluster.map_shared_rank(&slot, live ? lane : 0);
    const float pmd = live ? p->md : -INFINITY, pmt = live ? p->mt : -INFINITY;
    const double psd = live ? p->sd : 0.0, pst = live ? p->st : 0.0;
    const uint32_t pfl = live ? p->data_fl : 0u;
    const int phx = live ? p->has_x : 0;
    const float pedx = live ? p->ed_x : 0.f, petx = live ? p->et_x : 0.f;
    const float Md = warp_max(pmd), Mt = warp_max(pmt);
    const double fd = live ? exp((double)pmd - (double)Md) : 0.0;  // exp(m_r - M): rank weight factor
    const double ft = live ? exp((double)pmt - (double)Mt) : 0.0;
    const double wd = live ? psd * fd : 0.0, wt = live ? pst * ft : 0.0;
    const double Sd = __shfl_sync(0xffffffffu, warp_incl_scan_d(wd), 31);
    const double St = __shfl_sync(0xffffffffu, warp_incl_scan_d(wt), 31);
    const uint32_t fl = __reduce_or_sync(0xffffffffu, pfl);
    const unsigned xm = __ballot_sync(0xffffffffu, phx != 0);
    const int owner = xm ? __ffs(xm) - 1 : 0;
    const double pdx = __shfl_sync(0xffffffffu, (double)pedx * fd, owner) / Sd;
    const double ptx = __shfl_sync(0xffffffffu, (double)petx * ft, owner) / St;
    const double own_fd = __shfl_sync(0xffffffffu, fd, rank), own_ft = __shfl_sync(0xffffffffu, ft, rank);
    if (live) sh_wt[lane] = wt;
    if (lane == 0) {
      s_St = St;
      s_ft = own_ft;
      s_cd = (float)(own_fd / Sd);
      s_ct = (float)(own_ft / St);
      s_pdx = pdx;
      s_ptx = ptx;
      s_xfound = xm != 0;
      s_dfl = fl;
    }
  }
  __syncthreads();

  // ------------------------------------------------------------------ pass 3: TV and residual mass
  double Smin = 0.0, Z = 0.0;
  const bool phase_c = need_cstar || need_acc;
  const float cd = s_cd, ct = s_ct;
  if (phase_c) {
    float amin = 0.f, aq = 0.f;
    for (int i = tid; i < n; i += nthr) {
      const float pd = __fmul_rn(sd[i], cd), pt = __fmul_rn(st[i], ct);
      amin += fminf(pd, pt);
      aq += fmaxf(pt - pd, 0.f);
    }
    const double2 s2 = block_sum2((double)amin, (double)aq, sh_d);
    if (tid == 0) {
      slot.smin = s2.x;
      slot.sq = s2.y;
    }
    cluster.sync();  // (2) every CTA's (sum min, residual mass) is visible
    if (warp == 0) {
      const bool live = lane < CS;
      const Slot* p = cluster.map_shared_rank(&slot, live ? lane : 0);
      const double pm = live ? p->smin : 0.0, pq = live ? p->sq : 0.0;
      const double tm = __shfl_sync(0xffffffffu, warp_incl_scan_d(pm), 31);
      const double tq = __shfl_sync(0xffffffffu, warp_incl_scan_d(pq), 31);
      if (live) sh_wq[lane] = pq;
      if (lane == 0) {
        s_Smin = tm;
        s_Z = tq;
      }
    }
    __syncthreads();
    Smin = s_Smin;
    Z = s_Z;
  }

  // ------------------------------------------------------------------ pass 4: residual / bonus sample
  if (need_acc || need_bonus) {
    const bool use_q = need_acc && Z > 0.0;
    const double Wtot = use_q ? Z : s_St;
    const double t = (double)a.u_res[b] * Wtot;
    double P = 0.0;
    for (int r = 0; r < rank; ++r) P += use_q ? sh_wq[r] : sh_wt[r];
    const double Wr = use_q ? sh_wq[rank] : sh_wt[rank];
    const double Pn = P + Wr;
    int last_nz = -1;
    for (int r = 0; r < CS; ++r)
      if ((use_q ? sh_wq[r] : sh_wt[r]) > 0.0) last_nz = r;
    const bool cross = (Wr > 0.0) && (P <= t) && (t < Pn || rank == last_nz);
    if (cross) {  // uniform over the CTA
      const double fbonus = s_ft;  // element weights of the bonus row in units of exp(z - M_t)
      const int seg = (n + nthr - 1) / nthr;
      const int i0 = min(n, tid * seg), i1 = min(n, i0 + seg);
      double tsum = 0.0;
      for (int i = i0; i < i1; ++i)
        tsum += use_q ? (double)fmaxf(__fmul_rn(st[i], ct) - __fmul_rn(sd[i], cd), 0.f) : (double)st[i] * fbonus;
      const double incl = warp_incl_scan_d(tsum);
      double excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.0;
      if (lane == 31) sh_w[warp] = incl;
      if (tid == 0) s_pick = -1;
      __syncthreads();
      double wpre = P;
      for (int w = 0; w < warp; ++w) wpre += sh_w[w];
      const double pre = wpre + excl, nxt = wpre + incl;
      const bool last_nonempty = (i0 < i1) && (i1 == n);
      if (i0 < i1 && pre <= t && (t < nxt || last_nonempty)) {
        double R = pre, Rlast = pre, wlast = 0.0;
        int pick = -1, last = -1;
        double lo = 0.0, hi = 0.0;
        for (int i = i0; i < i1; ++i) {
          const double w =
              use_q ? (double)fmaxf(__fmul_rn(st[i], ct) - __fmul_rn(sd[i], cd), 0.f) : (double)st[i] * fbonus;
          if (w > 0.0) {
            last = i;
            Rlast = R;
            wlast = w;
            if (t < R + w) {
              pick = i;
              lo = R;
              hi = R + w;
              break;
            }
          }
          R += w;
        }
        if (pick < 0 && last >= 0) {
          pick = last;
          lo = Rlast;
          hi = Rlast + wlast;
        }
        if (pick >= 0) {
          s_pick = pick;
          s_lo = lo;
          s_hi = hi;
        }
      }
      __syncthreads();
      if (tid == 0) {
        int pick = s_pick;
        double lo = s_lo, hi = s_hi;
        if (pick < 0) {  // rounding left the threshold past every positive weight of the slice
          for (int i = n - 1; i >= 0; --i) {
            const double w =
                use_q ? (double)fmaxf(__fmul_rn(st[i], ct) - __fmul_rn(sd[i], cd), 0.f) : (double)st[i] * fbonus;
            if (w > 0.0) {
              pick = i;
              lo = hi = t;
              break;
            }
          }
        }
        uint32_t fl = 0;
        if ((t - lo) < 1e-6 * Wtot || (hi - t) < 1e-6 * Wtot) fl |= DSPARK_FLAG_SAMPLE_NEAR_TIE;
        if (need_acc && Z < 1e-3) fl |= DSPARK_FLAG_SMALL_RESIDUAL;
        Slot* s0 = cluster.map_shared_rank(&slot, 0);
        s0->cand = pick >= 0 ? v_beg + pick : -1;
        s0->cand_fl = fl;
      }
    }
  }
  cluster.sync();  // (3) the candidate token is in rank 0's slot

  // ------------------------------------------------------------------ row results (rank 0)
  // no distributed shared memory access past this point: peers may have exited
  if (rank == 0 && tid == 0) {
    uint32_t dfl = s_dfl;
    if (timed_out) dfl |= DSPARK_FLAG_DEVICE_TIMEOUT;
    if (need_cstar) {
      const double cs = (Z <= 0.5) ? 1.0 - Z : Smin;
      a.c_star[(size_t)b * a.gamma + kk] = (float)cs;
    }
    if (need_acc || need_bonus) {
      const size_t ri = (size_t)b * (a.gamma + 1) + kk;
      uint32_t rfl = slot.cand_fl;
      if (need_acc) {
        const int xk = a.x[(size_t)b * a.gamma + kk];
        int acc = 0;
        if ((unsigned)xk >= (unsigned)a.V || !s_xfound) {
          dfl |= DSPARK_FLAG_TOKEN_RANGE;
        } else {
          const double pd = s_pdx, pt = s_ptx;
          const double u = (double)a.u_acc[(size_t)b * a.gamma + kk];
          acc = (u * pd < pt) ? 1 : 0;
          if (pd > 0.0 && fabs(u - pt / pd) < 1e-6) rfl |= DSPARK_FLAG_ACCEPT_NEAR_TIE;
        }
        a.row_acc[ri] = acc;
      }
      int cand = slot.cand;
      if (cand < 0 || cand >= a.V) {
        dfl |= DSPARK_FLAG_NONFINITE;
        cand = min(max(cand, 0), a.V - 1);
      }
      a.row_cand[ri] = cand;
      a.row_fl[ri] = rfl;
    }
    if (dfl && a.flags) atomicOr(a.flags + b, dfl);
  }
}

// ============================================================================ persistent verify (T > 0)
//
// Each cluster walks the rows cid, cid + ncl, ... with the row slices double-buffered in
// shared memory: the bulk copies of row i+1 are in flight while row i is computed.  Per row:
//   pass 1  each thread takes its float4s of l_d and l_t into registers, z = l * (1/T), its own
//           max m_th and e = exp(z - m_th), sum e  (one pass, no block barrier in between);
//           a warp / block combine of (max, sum) pairs gives the CTA's pair;
//   S1      cluster barrier; warp 0 folds the CS pairs into M, S (fp64, rank order);
//   pass 2  p = e * exp(m_th - M) / S; sum min(p_d, p_t), sum max(0, p_t - p_d); the sample
//           weights (residual q and target p_t) are written back to the row's buffer;
//   S2      cluster barrier (only when TV labels or a residual are needed); fold the sums;
//   pass 3  the CTA holding u_res * W scans its slice in fp64 and writes the token into rank 0's
//           slot; rank 0 commits the row after the next barrier (S1 of the next row).

struct __align__(16) PSlot {
  double s_d, s_t;    // CTA sums of exp(z - m_cta)
  double smin, sq;    // CTA sums of min(p_d, p_t) and max(0, p_t - p_d)
  float m_d, m_t;     // CTA maxima of z
  float ex_d, ex_t;   // drafted token: exp(z - m_th) of its owner thread ...
  float mx_d, mx_t;   // ... and that thread's maxima
  int has_x;
  uint32_t data_fl;
  int cand;           // sampled token, written into rank 0's slot by the CTA holding it
  uint32_t cand_fl;
};

__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (max, sum-of-exp) pair combine; the sums are relative to their own maxima.
__device__ __forceinline__ void ms_combine(float& m, float& s, float m2, float s2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) {
    s = 0.f;
  } else {
    s = s * ex2a((m - M) * kLog2e) + s2 * ex2a((m2 - M) * kLog2e);
  }
  m = M;
}

struct RowNeed {
  int b, kk, Lb;
  bool cstar, acc, bonus, d, t;
};

__device__ __forceinline__ RowNeed row_need(const VerifyArgs& a, long long row) {
  RowNeed r;
  r.b = (int)(row / a.rows_per_req);
  r.kk = (int)(row - (long long)r.b * a.rows_per_req);
  r.Lb = a.gamma;
  if (a.do_verify && a.L) r.Lb = min(max(a.L[r.b], 0), a.gamma);
  r.cstar = (a.c_star != nullptr) && r.kk < a.gamma && (!a.lt_off || r.kk <= r.Lb);
  r.acc = a.do_verify && r.kk < r.Lb;
  r.bonus = a.do_verify && r.kk == r.Lb;
  r.d = r.cstar || r.acc;
  r.t = r.d || r.bonus;
  return r;
}

template <int NI, int NBUF>
__global__ void __launch_bounds__(512, 1) verify_rows_pc(VerifyArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.x / CS, ncl = gridDim.x / CS;
  const int tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31, nw = nthr >> 5;

  extern __shared__ __align__(16) float psm[];  // [NBUF][2][Vc]: draft then target slice
  __shared__ PSlot slot[2];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ float4 sh_ms[16];       // per warp: (m_d, s_d, m_t, s_t)
  __shared__ double2 sh_d2[16];
  __shared__ double sh_wq[16], sh_wt[16], sh_w[16];
  __shared__ float s_Md, s_Mt;
  __shared__ double s_iSd, s_iSt, s_pdx, s_ptx, s_Smin, s_Z, s_WtT;
  __shared__ int s_xfound, s_pick;
  __shared__ uint32_t s_dfl;
  __shared__ double s_lo, s_hi;

  const int v_beg = rank * a.Vc;
  const int n = max(0, min(a.V, v_beg + a.Vc) - v_beg);
  const int n4 = n >> 2;  // the bulk path needs V % 4 == 0, so n % 4 == 0
  const long long nrows = (long long)a.B * a.rows_per_req;
  const float inv_T = a.inv_T;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    for (int q = 0; q < 2; ++q) {
      slot[q].cand = -1;
      slot[q].cand_fl = 0;
      slot[q].data_fl = 0;
      slot[q].has_x = 0;
    }
  }
  __syncthreads();

  uint32_t uses[2] = {0u, 0u}, par[2] = {0u, 0u};
  bool loaded[2] = {false, false};
  // issue the slices of `row` into buffer j; identical bookkeeping in every thread
  auto issue = [&](long long row, int j) {
    const RowNeed rn = row_need(a, row);
    loaded[j] = rn.t && n > 0;
    if (!loaded[j]) return;
    par[j] = uses[j] & 1u;
    ++uses[j];
    if (tid == 0) {
      float* sd = psm + (size_t)j * 2 * a.Vc;
      const uint32_t bytes = (uint32_t)n * 4u;
      const size_t rowd = (size_t)rn.kk * a.ld_sk + (size_t)rn.b * a.ld_sb + v_beg;
      const size_t rowt = lt_row_index(a.lt_off, a.lt_nrows, a.lt_rows, rn.b, rn.kk) * a.V + v_beg;
      mbar_arrive_expect_tx(&bar[j], rn.d ? 2u * bytes : bytes);
      if (rn.d) bulk_g2s(sd, a.ld + rowd, bytes, &bar[j]);
      bulk_g2s(sd + a.Vc, a.lt + rowt, bytes, &bar[j]);
    }
  };

  // rank 0 commits a row once its sampled token is visible (after the next cluster barrier)
  bool pend = false;
  int p_b = 0, p_kk = 0, p_Lb = 0, p_acc = 0, p_j = 0;
  uint32_t p_fl = 0, p_dfl = 0;
  bool p_sample = false;
  auto commit = [&]() {
    if (!pend) return;
    pend = false;
    uint32_t dfl = p_dfl;
    if (p_sample) {
      const size_t ri = (size_t)p_b * (a.gamma + 1) + p_kk;
      int cand = slot[p_j].cand;
      if (cand < 0 || cand >= a.V) {
        dfl |= DSPARK_FLAG_NONFINITE;
        cand = min(max(cand, 0), a.V - 1);
      }
      if (p_kk < p_Lb) a.row_acc[ri] = p_acc;
      a.row_cand[ri] = cand;
      a.row_fl[ri] = p_fl | slot[p_j].cand_fl;
      slot[p_j].cand = -1;
      slot[p_j].cand_fl = 0;
    }
    if (dfl && a.flags) atomicOr(a.flags + p_b, dfl);
  };

  bool timed_out = false;
  int processed = 0;
  long long row = cid;
  if (row < nrows) issue(row, 0);
  for (int it = 0; row < nrows; row += ncl, ++it) {
    const int j = NBUF == 2 ? (it & 1) : 0;  // shared-memory buffer of this row
    const RowNeed rn = row_need(a, row);
    const long long nxt = row + ncl;
    if (NBUF == 2 && nxt < nrows) issue(nxt, j ^ 1);  // its last reader passed the barrier that ended row it-1
    if (!rn.t) {
      if (NBUF == 1 && nxt < nrows) {
        __syncthreads();
        issue(nxt, 0);
      }
      continue;
    }
    // exchange slot: alternates over the rows this cluster processes (skipped rows have no
    // cluster barrier, so the slot of the previous processed row is the one reset at S1)
    const int sj = processed & 1;
    ++processed;
    if (loaded[j] && !mbar_wait(&bar[j], par[j])) timed_out = true;
    float* sd = psm + (size_t)j * 2 * a.Vc;
    float* st = sd + a.Vc;
    float4* sd4 = reinterpret_cast<float4*>(sd);
    float4* st4 = reinterpret_cast<float4*>(st);

    // ---------------------------------------------------------------- pass 1 (registers)
    float4 ev_d[NI], ev_t[NI];
    float mthd = -INFINITY, mtht = -INFINITY;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      const int f = tid + i * nthr;
      float4 t4 = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY), d4 = t4;
      if (f < n4) {
        t4 = st4[f];
        t4 = make_float4(__fmul_rn(t4.x, inv_T), __fmul_rn(t4.y, inv_T), __fmul_rn(t4.z, inv_T), __fmul_rn(t4.w, inv_T));
        if (rn.d) {
          d4 = sd4[f];
          d4 = make_float4(__fmul_rn(d4.x, inv_T), __fmul_rn(d4.y, inv_T), __fmul_rn(d4.z, inv_T), __fmul_rn(d4.w, inv_T));
        }
      }
      ev_t[i] = t4;
      ev_d[i] = d4;
      mtht = fmaxf(mtht, fmaxf(fmaxf(t4.x, t4.y), fmaxf(t4.z, t4.w)));
      mthd = fmaxf(mthd, fmaxf(fmaxf(d4.x, d4.y), fmaxf(d4.z, d4.w)));
    }
    float sthd = 0.f, stht = 0.f;
    {
      // a thread with no finite maximum (no elements, or all -inf) contributes e = 0
      const float cd = mthd == -INFINITY ? 0.f : mthd * kLog2e, ct = mtht == -INFINITY ? 0.f : mtht * kLog2e;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        float4& t4 = ev_t[i];
        t4.x = ex2a(fmaf(t4.x, kLog2e, -ct));
        t4.y = ex2a(fmaf(t4.y, kLog2e, -ct));
        t4.z = ex2a(fmaf(t4.z, kLog2e, -ct));
        t4.w = ex2a(fmaf(t4.w, kLog2e, -ct));
        stht += (t4.x + t4.y) + (t4.z + t4.w);
        float4& d4 = ev_d[i];
        d4.x = ex2a(fmaf(d4.x, kLog2e, -cd));
        d4.y = ex2a(fmaf(d4.y, kLog2e, -cd));
        d4.z = ex2a(fmaf(d4.z, kLog2e, -cd));
        d4.w = ex2a(fmaf(d4.w, kLog2e, -cd));
        sthd += (d4.x + d4.y) + (d4.z + d4.w);
      }
    }
    const bool nonfin = (mtht == INFINITY) || (mthd == INFINITY) || isnan(stht) || isnan(sthd);
    // drafted token: its owner thread reports e and its thread maxima
    if (rn.acc) {
      const int xk = a.x[(size_t)rn.b * a.gamma + rn.kk];
      const int off = xk - v_beg;
      if (off >= 0 && off < n && ((off >> 2) % nthr) == tid) {
        const int i = (off >> 2) / nthr, c = off & 3;
        float exd = 0.f, ext = 0.f;
#pragma unroll
        for (int ii = 0; ii < NI; ++ii)
          if (ii == i) {
            exd = c == 0 ? ev_d[ii].x : c == 1 ? ev_d[ii].y : c == 2 ? ev_d[ii].z : ev_d[ii].w;
            ext = c == 0 ? ev_t[ii].x : c == 1 ? ev_t[ii].y : c == 2 ? ev_t[ii].z : ev_t[ii].w;
          }
        slot[sj].ex_d = exd;
        slot[sj].ex_t = ext;
        slot[sj].mx_d = mthd;
        slot[sj].mx_t = mtht;
        slot[sj].has_x = 1;
      }
    }
    // CTA (max, sum) pairs
    {
      float md = mthd, sdd = sthd, mt = mtht, stt = stht;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ms_combine(md, sdd, __shfl_xor_sync(0xffffffffu, md, o), __shfl_xor_sync(0xffffffffu, sdd, o));
        ms_combine(mt, stt, __shfl_xor_sync(0xffffffffu, mt, o), __shfl_xor_sync(0xffffffffu, stt, o));
      }
      const unsigned nf = __ballot_sync(0xffffffffu, nonfin);
      if (lane == 0) sh_ms[warp] = make_float4(md, sdd, mt, stt);
      if (lane == 0 && nf) atomicOr(&slot[sj].data_fl, DSPARK_FLAG_NONFINITE);
      __syncthreads();
      if (warp == 0) {
        float4 v = lane < nw ? sh_ms[lane] : make_float4(-INFINITY, 0.f, -INFINITY, 0.f);
        const float Md = warp_max(v.x), Mt = warp_max(v.z);
        const double wd = (v.x == -INFINITY) ? 0.0 : (double)v.y * (double)ex2a((v.x - Md) * kLog2e);
        const double wt = (v.z == -INFINITY) ? 0.0 : (double)v.w * (double)ex2a((v.z - Mt) * kLog2e);
        const double Sd = __shfl_sync(0xffffffffu, warp_incl_scan_d(wd), 31);
        const double St = __shfl_sync(0xffffffffu, warp_incl_scan_d(wt), 31);
        if (lane == 0) {
          slot[sj].m_d = Md;
          slot[sj].m_t = Mt;
          slot[sj].s_d = Sd;
          slot[sj].s_t = St;
        }
      }
    }
    cluster.sync();  // S1: every CTA's (max, sum) pair, and the previous row's token, are visible
    if (rank == 0 && tid == 0) commit();
    if (warp == 0) {
      const bool live = lane < CS;
      const PSlot* p = cluster.map_shared_rank(&slot[sj], live ? lane : 0);
      const float pmd = live ? p->m_d : -INFINITY, pmt = live ? p->m_t : -INFINITY;
      const double psd = live ? p->s_d : 0.0, pst = live ? p->s_t : 0.0;
      const uint32_t pfl = live ? p->data_fl : 0u;
      const int phx = live ? p->has_x : 0;
      const float pexd = live ? p->ex_d : 0.f, pext = live ? p->ex_t : 0.f;
      const float pmxd = live ? p->mx_d : -INFINITY, pmxt = live ? p->mx_t : -INFINITY;
      const float Md = warp_max(pmd), Mt = warp_max(pmt);
      const double wd = (pmd == -INFINITY) ? 0.0 : psd * exp((double)pmd - (double)Md);
      const double wt = (pmt == -INFINITY) ? 0.0 : pst * exp((double)pmt - (double)Mt);
      const double Sd = __shfl_sync(0xffffffffu, warp_incl_scan_d(wd), 31);
      const double St = __shfl_sync(0xffffffffu, warp_incl_scan_d(wt), 31);
      const uint32_t fl = __reduce_or_sync(0xffffffffu, pfl);
      const unsigned xm = __ballot_sync(0xffffffffu, phx != 0);
      const int owner = xm ? __ffs(xm) - 1 : 0;
      const double pdx = (double)pexd * exp((double)pmxd - (double)Md) / Sd;
      const double ptx = (double)pext * exp((double)pmxt - (double)Mt) / St;
      const double wt_norm = wt / St;  // this rank's target probability mass
      const double WtT = __shfl_sync(0xffffffffu, warp_incl_scan_d(live ? wt_norm : 0.0), 31);
      if (live) sh_wt[lane] = wt_norm;
      if (lane == 0) {
        s_Md = Md;
        s_Mt = Mt;
        s_iSd = 1.0 / Sd;
        s_iSt = 1.0 / St;
        s_WtT = WtT;
        s_dfl = fl;
        s_xfound = xm != 0;
      }
      const double pdx0 = __shfl_sync(0xffffffffu, pdx, owner), ptx0 = __shfl_sync(0xffffffffu, ptx, owner);
      if (lane == 0) {
        s_pdx = pdx0;
        s_ptx = ptx0;
      }
    }
    __syncthreads();
    if (tid == 0) {  // the other slot was last read before this S1: ready for the next row
      slot[sj ^ 1].data_fl = 0;
      slot[sj ^ 1].has_x = 0;
    }

    // ---------------------------------------------------------------- pass 2: probabilities
    const bool sample = rn.acc || rn.bonus;
    const bool phase_c = rn.cstar || rn.acc;
    const float fd = (rn.d && mthd != -INFINITY) ? (float)((double)ex2a((mthd - s_Md) * kLog2e) * s_iSd) : 0.f;
    const float ft = (mtht != -INFINITY) ? (float)((double)ex2a((mtht - s_Mt) * kLog2e) * s_iSt) : 0.f;
    double Smin = 0.0, Z = 0.0;
    if (phase_c || sample) {
      float amin = 0.f, aq = 0.f;
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const int f = tid + i * nthr;
        if (f < n4) {
          const float4 d4 = ev_d[i], t4 = ev_t[i];
          const float4 pd = make_float4(__fmul_rn(d4.x, fd), __fmul_rn(d4.y, fd), __fmul_rn(d4.z, fd), __fmul_rn(d4.w, fd));
          const float4 pt = make_float4(__fmul_rn(t4.x, ft), __fmul_rn(t4.y, ft), __fmul_rn(t4.z, ft), __fmul_rn(t4.w, ft));
          const float4 q = make_float4(fmaxf(pt.x - pd.x, 0.f), fmaxf(pt.y - pd.y, 0.f), fmaxf(pt.z - pd.z, 0.f),
                                       fmaxf(pt.w - pd.w, 0.f));
          amin += (fminf(pd.x, pt.x) + fminf(pd.y, pt.y)) + (fminf(pd.z, pt.z) + fminf(pd.w, pt.w));
          aq += (q.x + q.y) + (q.z + q.w);
          if (sample) {
            sd4[f] = q;
            st4[f] = pt;
          }
        }
      }
      if (phase_c) {
        double m2 = warp_sum_d((double)amin), q2 = warp_sum_d((double)aq);
        if (lane == 0) sh_d2[warp] = make_double2(m2, q2);
        __syncthreads();
        if (tid == 0) {
          double tm = 0.0, tq = 0.0;
          for (int w = 0; w < nw; ++w) {
            tm += sh_d2[w].x;
            tq += sh_d2[w].y;
          }
          slot[sj].smin = tm;
          slot[sj].sq = tq;
        }
        cluster.sync();  // S2
        if (warp == 0) {
          const bool live = lane < CS;
          const PSlot* p = cluster.map_shared_rank(&slot[sj], live ? lane : 0);
          const double pm = live ? p->smin : 0.0, pq = live ? p->sq : 0.0;
          const double tm = __shfl_sync(0xffffffffu, warp_incl_scan_d(pm), 31);
          const double tq = __shfl_sync(0xffffffffu, warp_incl_scan_d(pq), 31);
          if (live) sh_wq[lane] = pq;
          if (lane == 0) {
            s_Smin = tm;
            s_Z = tq;
          }
        }
      }
      __syncthreads();
      if (phase_c) {
        Smin = s_Smin;
        Z = s_Z;
      }
    }

    // ---------------------------------------------------------------- pass 3: residual / bonus sample
    if (sample) {
      const bool use_q = rn.acc && Z > 0.0;
      const double* W = use_q ? sh_wq : sh_wt;
      const float* wbuf = use_q ? sd : st;
      double Wtot = 0.0;
      for (int r = 0; r < CS; ++r) Wtot += W[r];
      const double t = (double)a.u_res[rn.b] * Wtot;
      double P = 0.0;
      for (int r = 0; r < rank; ++r) P += W[r];
      const double Wr = W[rank];
      const double Pn = P + Wr;
      int last_nz = -1;
      for (int r = 0; r < CS; ++r)
        if (W[r] > 0.0) last_nz = r;
      const bool cross = (Wr > 0.0) && (P <= t) && (t < Pn || rank == last_nz);
      if (cross) {  // uniform over the CTA
        const int seg = (n + nthr - 1) / nthr;
        const int i0 = min(n, tid * seg), i1 = min(n, i0 + seg);
        double tsum = 0.0;
        for (int i = i0; i < i1; ++i) tsum += (double)wbuf[i];
        const double incl = warp_incl_scan_d(tsum);
        double excl = __shfl_up_sync(0xffffffffu, incl, 1);
        if (lane == 0) excl = 0.0;
        if (lane == 31) sh_w[warp] = incl;
        if (tid == 0) s_pick = -1;
        __syncthreads();
        double wpre = P;
        for (int w = 0; w < warp; ++w) wpre += sh_w[w];
        const double pre = wpre + excl, nx = wpre + incl;
        const bool last_nonempty = (i0 < i1) && (i1 == n);
        if (i0 < i1 && pre <= t && (t < nx || last_nonempty)) {
          double R = pre, Rlast = pre, wlast = 0.0, lo = 0.0, hi = 0.0;
          int pick = -1, last = -1;
          for (int i = i0; i < i1; ++i) {
            const double w = (double)wbuf[i];
            if (w > 0.0) {
              last = i;
              Rlast = R;
              wlast = w;
              if (t < R + w) {
                pick = i;
                lo = R;
                hi = R + w;
                break;
              }
            }
            R += w;
          }
          if (pick < 0 && last >= 0) {
            pick = last;
            lo = Rlast;
            hi = Rlast + wlast;
          }
          if (pick >= 0) {
            s_pick = pick;
            s_lo = lo;
            s_hi = hi;
          }
        }
        __syncthreads();
        if (tid == 0) {
          int pick = s_pick;
          double lo = s_lo, hi = s_hi;
          if (pick < 0) {  // rounding left the threshold past every positive weight of the slice
            for (int i = n - 1; i >= 0; --i)
              if (wbuf[i] > 0.f) {
                pick = i;
                lo = hi = t;
                break;
              }
          }
          uint32_t fl = 0;
          if ((t - lo) < 1e-6 * Wtot || (hi - t) < 1e-6 * Wtot) fl |= DSPARK_FLAG_SAMPLE_NEAR_TIE;
          if (rn.acc && Z < 1e-3) fl |= DSPARK_FLAG_SMALL_RESIDUAL;
          PSlot* s0 = cluster.map_shared_rank(&slot[sj], 0);
          s0->cand = pick >= 0 ? v_beg + pick : -1;
          s0->cand_fl = fl;
        }
      }
    }

    // ---------------------------------------------------------------- row results (rank 0)
    if (rank == 0 && tid == 0) {
      uint32_t dfl = s_dfl | (timed_out ? DSPARK_FLAG_DEVICE_TIMEOUT : 0u);
      if (rn.cstar) a.c_star[(size_t)rn.b * a.gamma + rn.kk] = (float)((Z <= 0.5) ? 1.0 - Z : Smin);
      uint32_t rfl = 0;
      int acc = 0;
      if (rn.acc) {
        const int xk = a.x[(size_t)rn.b * a.gamma + rn.kk];
        if ((unsigned)xk >= (unsigned)a.V || !s_xfound) {
          dfl |= DSPARK_FLAG_TOKEN_RANGE;
        } else {
          const double u = (double)a.u_acc[(size_t)rn.b * a.gamma + rn.kk];
          acc = (u * s_pdx < s_ptx) ? 1 : 0;
          if (s_pdx > 0.0 && fabs(u - s_ptx / s_pdx) < 1e-6) rfl |= DSPARK_FLAG_ACCEPT_NEAR_TIE;
        }
      }
      pend = true;
      p_b = rn.b;
      p_kk = rn.kk;
      p_Lb = rn.Lb;
      p_acc = acc;
      p_j = sj;
      p_fl = rfl;
      p_dfl = dfl;
      p_sample = sample;
      if (!sample) commit();  // nothing to wait for
    }
    __syncthreads();  // every reader of buffer j is done: it may be refilled
    if (NBUF == 1 && nxt < nrows) issue(nxt, 0);
  }
  cluster.sync();  // the last row's token is visible; no shared-memory access across CTAs after this
  if (rank == 0 && tid == 0) commit();
  if (timed_out && a.status) atomicOr(a.status, (uint32_t)DSPARK_ETIMEOUT);
}

// ============================================================================ host side

// Per-row kernels need the first part; the streaming kernels (the default with a workspace)
// the second.
size_t verify_rows_workspace_bytes(int B, int gamma) {
  const size_t rows = (size_t)B * (gamma + 1);
  return kWsHeader + 3 * align_up(rows * 4, 256) + align_up((size_t)B * 4, 256);
}

size_t verify_workspace_bytes(int B, int gamma, int V) {
  return std::max({verify_rows_workspace_bytes(B, gamma), stream_verify_workspace_bytes(B, gamma, V),
                   sliced_verify_workspace_bytes(B, gamma, V)});
}

// Cluster size: the smallest power of two whose per-CTA slices (ℓ_d and ℓ_t, fp32) fit the
// budget (80 KB by default, so two CTAs share an SM).  A requested size is raised if its
// slices would not fit in shared memory at all.
constexpr size_t kVerifySmemMax = 200 * 1024;

static int pick_cluster(int V, int requested) {
  const bool req = requested == 1 || requested == 2 || requested == 4 || requested == 8 || requested == 16;
  const size_t budget = req ? kVerifySmemMax : 80 * 1024;
  int cs = req ? requested : 1;
  while (cs < 16) {
    const size_t vc = align_up((size_t)(V + cs - 1) / cs, 4);
    if (8 * vc <= budget) break;
    cs *= 2;
  }
  return cs;
}

template <int NI, int NBUF>
static dspark_status launch_pc(const VerifyArgs& a, int cs, cudaStream_t stream) {
  auto kern = verify_rows_pc<NI, NBUF>;
  const size_t smem = (size_t)NBUF * 8 * a.Vc;
  cudaError_t rc = ensure_smem_attr((const void*)kern, smem);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(verify_rows_pc, smem): ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  if (cs > 8) {
    rc = ensure_nonportable_cluster((const void*)kern);
    if (rc != cudaSuccess) {
      set_error(std::string("cudaFuncSetAttribute(verify_rows_pc, cluster 16): ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  }
  const long long nrows = (long long)a.B * a.rows_per_req;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(512);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)cs);
  int ncl = 0;
  rc = cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg);
  if (rc != cudaSuccess || ncl <= 0) {
    (void)cudaGetLastError();
    return DSPARK_ENOTIMPL;
  }
  ncl = (int)std::min<long long>(ncl, nrows);
  cfg.gridDim = dim3((unsigned)(ncl * cs));
  rc = cudaLaunchKernelEx(&cfg, kern, a);
  if (rc != cudaSuccess) {
    set_error(std::string("verify launch (persistent, cluster ") + std::to_string(cs) + "): " + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

static dspark_status launch_finalize(const VerifyArgs& a, cudaStream_t stream) {
  if (!a.do_verify) return DSPARK_OK;
  verify_finalize<<<(a.B + 127) / 128, 128, 0, stream>>>(a);
  const cudaError_t rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("verify finalize launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

// double_buffer: rows double-buffered in shared memory (else single-buffered; also used when two
// buffers do not fit).  One CTA of 512 threads per SM either way.
static dspark_status launch_verify_persistent(const VerifyArgs& a, int cs, cudaStream_t stream, bool double_buffer) {
  const int per_thread = (a.Vc / 4 + 511) / 512;  // float4s per thread
  const bool two = double_buffer && (size_t)16 * a.Vc <= kVerifySmemMax;
  if (per_thread <= 1) return two ? launch_pc<1, 2>(a, cs, stream) : launch_pc<1, 1>(a, cs, stream);
  if (per_thread <= 2) return two ? launch_pc<2, 2>(a, cs, stream) : launch_pc<2, 1>(a, cs, stream);
  if (per_thread <= 4) return two ? launch_pc<4, 2>(a, cs, stream) : launch_pc<4, 1>(a, cs, stream);
  if (per_thread <= 6) return two ? launch_pc<6, 2>(a, cs, stream) : launch_pc<6, 1>(a, cs, stream);
  if (per_thread <= 8) return two ? launch_pc<8, 2>(a, cs, stream) : launch_pc<8, 1>(a, cs, stream);
  return DSPARK_ENOTIMPL;
}

dspark_status launch_verify(const VerifyCall& c) {
  if (c.do_verify && !c.per_row_only) {
    dspark_status st = launch_verify_stream(c);
    if (st != DSPARK_ENOTIMPL) return st;
    st = launch_verify_sliced(c);
    if (st != DSPARK_ENOTIMPL) return st;  // else: the per-row kernels below
  }
  VerifyArgs a{};
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
  a.rows_per_req = c.do_verify ? c.gamma + 1 : c.gamma;
  a.greedy = (c.T == 0.f) ? 1 : 0;
  a.inv_T = a.greedy ? 1.f : 1.f / c.T;
  a.do_verify = c.do_verify;
  a.c_star = c.c_star;
  a.n_acc = c.n_acc;
  a.y_out = c.y_out;
  a.flags = c.flags;
  cudaError_t rc;
  if (c.do_verify) {
    uint8_t* ws = static_cast<uint8_t*>(c.ws);
    const size_t rows = (size_t)c.B * (c.gamma + 1);
    a.status = reinterpret_cast<uint32_t*>(ws);
    a.row_acc = reinterpret_cast<int32_t*>(ws + kWsHeader);
    a.row_cand = reinterpret_cast<int32_t*>(ws + kWsHeader + align_up(rows * 4, 256));
    a.row_fl = reinterpret_cast<uint32_t*>(ws + kWsHeader + 2 * align_up(rows * 4, 256));
    a.counter = reinterpret_cast<int32_t*>(ws + kWsHeader + 3 * align_up(rows * 4, 256));
    rc = cudaMemsetAsync(ws, 0, kWsHeader, c.stream);
    if (rc != cudaSuccess) {
      set_error(std::string("cudaMemsetAsync: ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  }
  const Options opt = options();
  const int cs = pick_cluster(c.V, opt.verify_cluster);
  a.Vc = (int)align_up((size_t)(c.V + cs - 1) / cs, 4);
  if ((size_t)8 * a.Vc > kVerifySmemMax) {
    set_error("dspark_verify: V too large for one 16-CTA cluster per row (V <= 409600)");
    return DSPARK_ENOTIMPL;
  }
  a.bulk = (c.V % 4 == 0) && ((uintptr_t)c.lt % 16 == 0) && ((uintptr_t)c.ld % 16 == 0);
  if (!a.greedy && a.bulk && opt.verify_persistent) {
    dspark_status st = launch_verify_persistent(a, cs, c.stream, true);
    if (st == DSPARK_OK) st = launch_finalize(a, c.stream);
    if (st != DSPARK_ENOTIMPL) return st;  // else: no resident cluster fits; use the one-row-per-cluster kernel
  }
  const int nthr = a.Vc >= 4096 ? 512 : (a.Vc >= 1024 ? 256 : 128);
  const size_t smem = (size_t)8 * a.Vc;
  rc = ensure_smem_attr((const void*)verify_rows, smem);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(verify_rows, smem): ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  if (cs > 8) {
    rc = ensure_nonportable_cluster((const void*)verify_rows);
    if (rc != cudaSuccess) {
      set_error(std::string("cudaFuncSetAttribute(verify_rows, cluster 16): ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  }
  const long long nrows = (long long)c.B * a.rows_per_req;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nrows * cs));
  cfg.blockDim = dim3(nthr);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  rc = cudaLaunchKernelEx(&cfg, verify_rows, a);
  if (rc != cudaSuccess) {
    set_error(std::string("verify launch (cluster ") + std::to_string(cs) + "): " + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return launch_finalize(a, c.stream);
}

}  // namespace dspark

// ============================================================================ verify without allocation
//
// Some callers cannot hand this library a workspace at the moment they verify: a serving
// engine that has reserved almost all of HBM for its KV cache and permits no further
// cudaMalloc while decoding, or plugin code that receives raw device pointers from a host
// framework with no access to that framework's allocator.  dspark_verify_noalloc serves them
// from a fixed array in the library's own device memory instead of a caller workspace.
//
// It always runs the per-row cluster kernels (verify_rows_pc / verify_rows + verify_finalize):
// their scratch is a few words per row and request, so a fixed array covers every size up to
// the limits below, whatever V is.  The streaming kernels keep per-tile records that grow with
// V and are never used here.
//
// The array below is that scratch.  Every GPU that loads the library holds it until the
// process exits.  In host code its name is only a host-side stand-in, so its device address
// is looked up with cudaGetSymbolAddress once per device and CUDA context, with that device
// current (the first call on a device does this, which is why that first call should come
// before any stream capture; a call after the context was destroyed and recreated looks it up
// again).  All calls share the array: each call clears the words that must start at zero, and
// calls whose kernels overlap on the GPU race on it.

namespace dspark {

constexpr int kNoAllocMaxRows = 16384;  // B * (gamma + 1)
constexpr int kNoAllocMaxB = 4096;
constexpr size_t kNoAllocScratchBytes = kWsHeader + 3 * (size_t)kNoAllocMaxRows * 4 + (size_t)kNoAllocMaxB * 4;

static __device__ __align__(256) uint8_t g_verify_scratch[kNoAllocScratchBytes];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

static CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

static dspark_status verify_scratch(void** ptr) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  static CUcontext ctx_of[64] = {nullptr};
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess || dev < 0 || dev >= 64) {
    set_error(std::string("dspark_verify_noalloc: cudaGetDevice: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  CUcontext ctx = nullptr;
  const CtxGetCurrentFn cur = ctx_get_current_fn();
  if (cur) (void)cur(&ctx);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || !ctx || ctx_of[dev] != ctx) {
    void* p = nullptr;
    rc = cudaGetSymbolAddress(&p, g_verify_scratch);  // also makes the device's primary context current
    if (rc != cudaSuccess || !p) {
      set_error(std::string("dspark_verify_noalloc: cudaGetSymbolAddress: ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
    if (!ctx && cur) (void)cur(&ctx);
    addr[dev] = p;
    ctx_of[dev] = ctx;
  }
  *ptr = addr[dev];
  return DSPARK_OK;
}

}  // namespace dspark

extern "C" int dspark_verify_noalloc(const float* ld, const float* lt, const int32_t* x, const int32_t* L,
                                     const float* u_acc, const float* u_res, int B, int gamma, int V, float T,
                                     int ld_layout, int32_t* n_acc, int32_t* y_out, float* c_star, uint32_t* flags,
                                     void* stream) {
  using namespace dspark;
  auto einval = [](const char* msg) {
    set_error(msg);
    return (int)DSPARK_EINVAL;
  };
  if (!ld || !lt || !x || !n_acc || !y_out || !flags) return einval("dspark_verify_noalloc: null pointer");
  if (T != 0.f && (!u_acc || !u_res)) return einval("dspark_verify_noalloc: u_acc and u_res are required when T > 0");
  if (B <= 0 || V < 2) return einval("dspark_verify_noalloc: B must be >= 1 and V >= 2");
  if (gamma < 1 || gamma > kMaxGamma) return einval("dspark_verify_noalloc: gamma must be in [1, 64]");
  if (!(T >= 0.f) || std::isinf(T)) return einval("dspark_verify_noalloc: T must be finite and >= 0");
  if (ld_layout != DSPARK_POSITION_MAJOR && ld_layout != DSPARK_REQUEST_MAJOR)
    return einval("dspark_verify_noalloc: ld_layout must be DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR");
  if (B > kNoAllocMaxB || (long long)B * (gamma + 1) > kNoAllocMaxRows)
    return einval("dspark_verify_noalloc: needs B <= 4096 and B*(gamma+1) <= 16384 (fixed scratch); use dspark_verify");
  if (verify_rows_workspace_bytes(B, gamma) > kNoAllocScratchBytes)  // holds within the limits above
    return einval("dspark_verify_noalloc: fixed scratch too small for these sizes");
  void* ws = nullptr;
  const dspark_status st = verify_scratch(&ws);
  if (st != DSPARK_OK) return st;
  VerifyCall c{ld, lt, x, L, u_acc, u_res, B, gamma, V, gamma + 1, T, ld_layout, 1, 1, n_acc, y_out, c_star, flags, ws,
               kNoAllocScratchBytes, (cudaStream_t)stream};
  return launch_verify(c);
}

// ============================================================================ flattened target block
//
// Row offsets and token tags of the flattened verify block (one CTA): request b owns rows
// off[b] .. off[b] + L_b, off being the exclusive prefix sum of L_b + 1 (L_b clamped to
// [0, gamma]); row off[b] + k carries the tag b*(gamma+1) + k, and the tags past the last row,
// up to the capacity B*(gamma+1), are -1.

namespace dspark {

__global__ void __launch_bounds__(1024) ragged_layout_kernel(const int32_t* L, int B, int gamma, int64_t* off,
                                                             int32_t* tags) {
  __shared__ long long sh[32];
  __shared__ long long s_carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    s_carry = 0;
    off[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < B; base += 1024) {
    const int b = base + tid;
    const long long v = b < B ? (long long)min(max(__ldg(L + b), 0), gamma) + 1 : 0;
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    long long incl = s_carry + x;
    for (int w = 0; w < warp; ++w) incl += sh[w];
    if (b < B) {
      off[b + 1] = incl;
      if (tags)
        for (int k = 0; k < (int)v; ++k) tags[incl - v + k] = b * (gamma + 1) + k;
    }
    __syncthreads();
    if (tid == 1023) s_carry = incl;  // the chunk's total plus the carry
    __syncthreads();
  }
  if (tags) {
    const long long cap = (long long)B * (gamma + 1);
    for (long long i = s_carry + tid; i < cap; i += 1024) tags[i] = -1;
  }
}

dspark_status launch_ragged_layout(const int32_t* L, int B, int gamma, int64_t* lt_off, int32_t* tags,
                                   cudaStream_t stream) {
  ragged_layout_kernel<<<1, 1024, 0, stream>>>(L, B, gamma, lt_off, tags);
  const cudaError_t rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("ragged layout launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

}  // namespace dspark
