// Prefix survival and the greedy hardware-aware prefix scheduler.
//
// [P3 "DSpark Speculative Decoding" §Confidence-Scheduled Verification: a_{r,j} = ∏_{i≤j} c_{r,i};
//  Algorithm 1 maximises Θ = τ·SPS(B) by extending verify lengths greedily along a]
// [P1 "DeepSeek V4-Pro DSpark 推测解码方案深度解析" §硬件感知与置信度自适应调度机制: every candidate
//  token of the batch is ranked by cumulative survival and added one at a time while expected
//  accepted tokens x hardware speed keeps rising; the global search runs on the GPU]
//
// One CTA of 1024 threads: running products per request (fp32, left to right), 64-bit keys
// (survival descending, then flat index b*gamma + j), sorted in shared memory -- by a bottom-up
// merge of the requests' runs when every confidence lies in [0, 1] (each run is then already
// sorted), else bitonically with warp shuffles for the short strides --, an fp64 block scan of
// the sorted survivals giving Θ(D) = (B + S(D)) * sps[D] for D = 0..D_max, the ARGMAX /
// EARLY_STOP choice, and per-request counts of the kept items.
//
// Asynchronous variant ([P1 §硬件感知与置信度自适应调度机制, last paragraph: the truncation of
// step t is decided from the confidence history of step t-2, so the global search stays inside
// the GPU pipeline with no host handshake and survives CUDA-graph replay]; [P3 production notes,
// "asynchronous": confidences two steps back predict the batch capacity K]): a small device ring
// carries the step counter and the search results of the last four steps.  The same launch reads
// the capacity K_t = D*_{t-2} from it, keeps the first K_t items of this step's own survival
// order, stores this step's D*_t for step t+2 and advances the counter, so a captured graph can
// replay step after step with the ring as its only state.

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dspark {

constexpr int kSchedThreads = 1024;
constexpr int kSchedWarps = kSchedThreads / 32;
constexpr int kMergeMaxKeys = 8192;  // two key buffers of 64 KB

struct SchedArgs {
  const float* c;
  const double* sps;
  int B, gamma, D_max, mode, P;
  int P2;  // second key buffer for the merge sort (0: bitonic sort only)
  int32_t* L_out;
  float* a_out;
  double* theta_out;
  uint32_t* flags;
  T2Ring* ring;  // asynchronous (t-2) mode when set
  int K_init;    // capacity of steps 0 and 1 (< 0: D_max)
  int32_t* K_out;
};

// Survival descending -> ascending 32-bit key; -0 ranks as +0, NaN ranks last.
__device__ __forceinline__ uint32_t desc_key(float a) {
  if (isnan(a)) return 0xFFFFFFFFu;
  if (a == 0.f) a = 0.f;
  const uint32_t u = __float_as_uint(a);
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~ord;
}

__device__ __forceinline__ float key_value(uint64_t key) {
  const uint32_t ord = ~(uint32_t)(key >> 32);
  const uint32_t u = (ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord;
  return __uint_as_float(u);
}

__global__ void __launch_bounds__(kSchedThreads, 1) schedule_kernel(SchedArgs s) {
  extern __shared__ __align__(16) uint64_t keys[];
  uint64_t* keys2 = keys + s.P;  // [P2]
  int* cnt = reinterpret_cast<int*>(keys + s.P + s.P2);
  __shared__ double sh_pre[kSchedWarps];
  __shared__ double sh_tot;
  __shared__ double sh_w[kSchedWarps];
  __shared__ double sh_best[kSchedWarps];
  __shared__ int sh_bestD[kSchedWarps];
  __shared__ int sh_stop[kSchedWarps];
  __shared__ int sh_tie[kSchedWarps];
  __shared__ int s_D;
  __shared__ double s_theta;
  __shared__ int s_K;          // asynchronous mode: capacity applied at this step
  __shared__ double s_thetaK;  // Θ(s_K) of this step's order
  __shared__ unsigned s_tieK;  // the decision that gave s_K was a near-tie
  __shared__ long long s_t;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = s.B, G = s.gamma, N = B * G, P = s.P, Dm = s.D_max;
  if (s.ring && tid == 0) {
    const long long t = s.ring->t;
    int K = t >= 2 ? s.ring->D[(t - 2) & 3] : (s.K_init < 0 ? Dm : s.K_init);
    s_K = max(0, min(K, Dm));
    s_tieK = t >= 2 ? s.ring->tie[(t - 2) & 3] : 0u;
    s_t = t;
    s_thetaK = (double)B * s.sps[0];
  }

  // ---------------------------------------------------------------- survival and keys
  // c is staged in shared memory (the key array's space) with coalesced loads; each request's
  // running product is then taken in place, left to right, and the keys are built afterwards.
  float* cs = reinterpret_cast<float*>(keys);  // N floats fit in the first N/2 keys
  for (int i = tid; i < N; i += kSchedThreads) cs[i] = s.c[i];
  __syncthreads();
  int any_bad = 0;
  for (int b = tid; b < B; b += kSchedThreads) {
    float prod = 1.f;
    bool bad = false;
    for (int j = 0; j < G; ++j) {
      const float cj = cs[b * G + j];
      bad |= !(cj >= 0.f && cj <= 1.f);
      prod = (j == 0) ? cj : __fmul_rn(prod, cj);
      cs[b * G + j] = prod;
    }
    if (bad && s.flags) atomicOr(s.flags + b, DSPARK_FLAG_CONF_RANGE);
    any_bad |= bad ? 1 : 0;
    cnt[b] = 0;
  }
  // with every confidence in [0, 1] each request's survivals are non-increasing (an fp32 product
  // with a factor <= 1 never exceeds the other factor), so its keys already form a sorted run
  const bool runs_sorted = __syncthreads_or(any_bad) == 0;
  constexpr int kMaxPer = kMaxScheduleItems / kSchedThreads;
  float av[kMaxPer];
#pragma unroll
  for (int m = 0; m < kMaxPer; ++m) {
    const int i = tid + m * kSchedThreads;
    av[m] = i < N ? cs[i] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < kMaxPer; ++m) {
    const int i = tid + m * kSchedThreads;
    if (i < P) keys[i] = i < N ? (((uint64_t)desc_key(av[m]) << 32) | (uint32_t)i) : ~0ull;
    if (i < N && s.a_out) s.a_out[i] = av[m];
  }
  __syncthreads();

  // ---------------------------------------------------------------- sort (ascending keys)
  // Sorted runs (every confidence in [0, 1]) and room for a second buffer: a bottom-up merge of
  // the B runs of gamma keys, each key placed at its run position plus its rank in the partner
  // run (a binary search; keys are distinct, so the merge keeps b ascending on equal survivals).
  // Otherwise a bitonic sort of all P keys in place.
  const uint64_t* ks = keys;
  if (runs_sorted && s.P2 > 0) {
    uint64_t* src = keys;
    uint64_t* dst = keys2;
    for (int w = G; w < N; w <<= 1) {
      for (int e = tid; e < N; e += kSchedThreads) {
        const int r = e / w, pos = e - r * w;
        const int pstart = (r ^ 1) * w;
        const int plen = max(0, min(pstart + w, N) - pstart);
        const uint64_t x = src[e];
        int lo = 0, hi = plen;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (src[pstart + mid] < x) lo = mid + 1;
          else hi = mid;
        }
        dst[(r & ~1) * w + pos + lo] = x;
      }
      __syncthreads();
      uint64_t* t = src;
      src = dst;
      dst = t;
    }
    ks = src;
  } else {
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        if (j >= 32 || P < 64) {
          for (int i = tid; i < P; i += kSchedThreads) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const uint64_t x = keys[i], y = keys[ixj];
              const bool up = (i & k) == 0;
              if ((x > y) == up) {
                keys[i] = y;
                keys[ixj] = x;
              }
            }
          }
          __syncthreads();
        } else {
          // strides 16..1 stay inside a warp: 32 consecutive keys per warp pass
          for (int base = warp * 32; base < P; base += kSchedThreads) {
            const int i = base + lane;
            uint64_t x = keys[i];
            for (int jj = j; jj > 0; jj >>= 1) {
              const uint64_t y = __shfl_xor_sync(0xffffffffu, x, jj);
              const bool up = (i & k) == 0;
              const bool lower = (lane & jj) == 0;
              const uint64_t mn = x < y ? x : y, mx = x < y ? y : x;
              x = (lower == up) ? mn : mx;
            }
            keys[i] = x;
          }
          __syncthreads();
          break;  // all strides below 32 handled
        }
      }
    }
  }

  // ---------------------------------------------------------------- Θ pass (twice: choose, then tie check)
  // The sorted survivals are scanned in chunks of kSchedThreads items; item i moves D from
  // i to i+1, so the thread owning it sees Θ(i) and Θ(i+1).
  // Block-wide scan step: the sum of the earlier warps' totals (plus the carry of earlier
  // chunks) for this thread's warp; the carry grows by the chunk's total.
  auto block_prefix = [&](double incl, double& carry_io) -> double {
    if (lane == 31) sh_w[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const double v = sh_w[lane];
      const double inc = warp_incl_scan_d(v);
      double ex = __shfl_up_sync(0xffffffffu, inc, 1);
      if (lane == 0) ex = 0.0;
      sh_pre[lane] = ex;
      if (lane == 31) sh_tot = inc;
    }
    __syncthreads();
    const double wpre = carry_io + sh_pre[warp];
    carry_io += sh_tot;
    return wpre;
  };
  const double theta0 = (double)B * s.sps[0];
  double best = theta0;
  int bestD = 0;
  int stop = Dm;  // EARLY_STOP: first d with Θ(d+1) <= Θ(d)
  for (int pass = 0; pass < 2; ++pass) {
    int tie = 0;
    double carry = 0.0;
    const int Dstar = pass ? s_D : 0;
    const double th_star = pass ? s_theta : 0.0;
    for (int base = 0; base < Dm; base += kSchedThreads) {
      const int i = base + tid;
      const double ai = (i < Dm) ? (double)key_value(ks[i]) : 0.0;
      const double incl = warp_incl_scan_d(ai);
      double excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.0;
      const double wpre = block_prefix(incl, carry);
      if (i < Dm) {
        const double th_lo = ((double)B + (wpre + excl)) * s.sps[i];      // Θ(i)
        const double th_hi = ((double)B + (wpre + incl)) * s.sps[i + 1];  // Θ(i+1)
        if (pass == 0) {
          if (th_hi > best) {
            best = th_hi;
            bestD = i + 1;
          }
          if (th_hi <= th_lo && i < stop) stop = i;
          if (s.ring && i + 1 == s_K) s_thetaK = th_hi;
        } else if (s.mode == DSPARK_SCHED_ARGMAX) {
          if (i + 1 != Dstar && fabs(th_hi - th_star) <= 1e-12 * fabs(th_star)) tie = 1;
        } else {
          if (i <= Dstar && i < Dm && fabs(th_hi - th_lo) <= 1e-12 * fabs(th_lo)) tie = 1;
        }
      }
    }
    if (pass == 0) {
      // argmax with the smallest D among equal Θ; first stop index
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int od = __shfl_xor_sync(0xffffffffu, bestD, o);
        if (ob > best || (ob == best && od < bestD)) {
          best = ob;
          bestD = od;
        }
        stop = min(stop, __shfl_xor_sync(0xffffffffu, stop, o));
      }
      if (lane == 0) {
        sh_best[warp] = best;
        sh_bestD[warp] = bestD;
        sh_stop[warp] = stop;
      }
      __syncthreads();
      if (tid == 0) {
        double bb = sh_best[0];
        int bd = sh_bestD[0], sp = sh_stop[0];
        for (int w = 1; w < kSchedWarps; ++w) {
          if (sh_best[w] > bb || (sh_best[w] == bb && sh_bestD[w] < bd)) {
            bb = sh_best[w];
            bd = sh_bestD[w];
          }
          sp = min(sp, sh_stop[w]);
        }
        if (s.mode == DSPARK_SCHED_ARGMAX) {
          s_D = bd;
          s_theta = bb;
        } else {
          s_D = sp;
          s_theta = 0.0;  // filled in below
        }
      }
      __syncthreads();
      if (s.mode != DSPARK_SCHED_ARGMAX) {
        // Θ(D*) for EARLY_STOP: recompute S(D*) serially from the sorted keys is O(D); use the
        // scan instead: the thread owning item D*-1 knows Θ(D*).
        const int Ds = s_D;
        double carry2 = 0.0;
        for (int base = 0; base < max(Ds, 1); base += kSchedThreads) {
          const int i = base + tid;
          const double ai = (i < Ds) ? (double)key_value(ks[i]) : 0.0;
          const double incl = warp_incl_scan_d(ai);
          const double wpre = block_prefix(incl, carry2);
          if (i == Ds - 1) s_theta = ((double)B + (wpre + incl)) * s.sps[Ds];
        }
        if (Ds == 0 && tid == 0) s_theta = theta0;
        __syncthreads();
      }
    } else {
      const int any = __any_sync(0xffffffffu, tie);
      if (lane == 0) sh_tie[warp] = any;
      __syncthreads();
      if (tid == 0) {
        int t = 0;
        for (int w = 0; w < kSchedWarps; ++w) t |= sh_tie[w];
        if (s.mode == DSPARK_SCHED_ARGMAX && s_D != 0 && fabs(theta0 - s_theta) <= 1e-12 * fabs(s_theta)) t = 1;
        sh_tie[0] = t;
      }
      __syncthreads();
    }
  }

  // ---------------------------------------------------------------- counts and outputs
  // synchronous mode keeps the first D* items; asynchronous mode the first K_t (= D*_{t-2})
  const int Ds = s.ring ? s_K : s_D;
  for (int i = tid; i < Ds; i += kSchedThreads) atomicAdd(&cnt[(int)(uint32_t)ks[i] / G], 1);
  __syncthreads();
  const bool near = s.ring ? s_tieK != 0 : sh_tie[0] != 0;
  for (int b = tid; b < B; b += kSchedThreads) {
    s.L_out[b] = cnt[b];
    if (near && s.flags) atomicOr(s.flags + b, DSPARK_FLAG_SCHED_NEAR_TIE);
  }
  if (tid == 0) {
    if (s.ring) {
      const int slot = (int)(s_t & 3);
      s.ring->D[slot] = s_D;
      s.ring->tie[slot] = sh_tie[0] ? 1u : 0u;
      s.ring->theta[slot] = s_theta;
      s.ring->K[slot] = s_K;
      s.ring->t = s_t + 1;
      s.theta_out[0] = s_thetaK;
      if (s.K_out) s.K_out[0] = s_K;
    } else {
      s.theta_out[0] = s_theta;
    }
  }
}

dspark_status launch_schedule(const ScheduleCall& c) {
  SchedArgs s{};
  s.c = c.c;
  s.sps = c.sps;
  s.B = c.B;
  s.gamma = c.gamma;
  s.D_max = c.D_max;
  s.mode = c.mode;
  int P = 64;
  while (P < c.B * c.gamma) P <<= 1;
  s.P = P;
  s.P2 = P <= kMergeMaxKeys ? P : 0;  // a second key buffer fits in shared memory
  s.L_out = c.L_out;
  s.a_out = c.a_out;
  s.theta_out = c.theta_out;
  s.flags = c.flags;
  s.ring = c.ring;
  s.K_init = c.K_init;
  s.K_out = c.K_out;
  const size_t smem = (size_t)(P + s.P2) * 8 + align_up((size_t)c.B * 4, 16);
  cudaError_t rc;
  if (smem > 48 * 1024) {
    rc = ensure_smem_attr((const void*)schedule_kernel, smem);
    if (rc != cudaSuccess) {
      set_error(std::string("cudaFuncSetAttribute(schedule_kernel): ") + cudaGetErrorString(rc));
      return DSPARK_ECUDA;
    }
  }
  schedule_kernel<<<1, kSchedThreads, smem, c.stream>>>(s);
  rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("schedule launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

}  // namespace dspark
