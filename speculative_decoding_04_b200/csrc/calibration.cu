// Confidence calibration: sequential temperature scaling (STS) fitted on a validation set, its
// application to a round's confidences, and the expected calibration error (ECE).
//
// [P1 "DeepSeek V4-Pro DSpark 推测解码方案深度解析" §硬件感知与置信度自适应调度机制: the confidence
//  head is over-confident; a 1-D grid search per candidate position on a validation set finds the
//  temperature that calibrates it (ECE from 3-8 % to about 1 %); temperature scaling keeps the
//  order of the confidences]
// [P3 "DSpark Speculative Decoding" §Confidence-Scheduled Verification: STS calibrates the
//  cumulative product position by position]
//
// A confidence is scaled as sigma(logit(c) / tau) in fp64 (c clamped to [0, 1], NaN as 0).
// Position k is fitted after positions 0..k-1: for every grid temperature the calibrated survival
// a'_k = a'_{k-1} * sigma(logit(c_k) / tau) of every sample goes into one of M equal-width bins,
// each bin summing (s - a'_k) with s = 1 when the sample's first k+1 positions were accepted; the
// ECE of that temperature is sum over bins of |sum| / N.  The raw cumulative products (tau = 1
// everywhere) get the same histogram for the before/after comparison.
//
// Two launches per position: sts_hist (grid-stride over the samples, histograms of all grid
// temperatures in shared memory, flushed with fp64 atomics) and sts_select (one CTA: the ECE of
// every temperature and the first minimum).  sts_hist of position k first extends each sample's
// running products by position k-1 with the temperature sts_select just chose, so the samples'
// state stays in two fp64 arrays of the workspace.

#include <algorithm>
#include <cfloat>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace dspark {

namespace {

constexpr int kStsThreads = 256;

struct StsArgs {
  const float* c;      // [N][gamma]
  const int32_t* n;    // [N] accepted counts
  long long N;
  int gamma, J, M;
  const double* grid;  // [J]
  double* a_cal;       // [N] calibrated running product up to the previous position
  double* a_raw;       // [N] raw running product up to the previous position
  double* hist;        // [gamma][J + 1][M]: per (temperature, bin) sum of (s - p); row J: raw products
  double* tau;         // [gamma]
  int32_t* index;      // [gamma]
  double* ece_raw;     // [gamma]
  double* ece_cal;     // [gamma]
  double* curve;       // [gamma][J] or null
};

__device__ __forceinline__ double sts_clamp(float c) {
  const double v = (double)c;
  return v > 0.0 ? (v < 1.0 ? v : 1.0) : 0.0;  // NaN compares false: 0
}

// sigma(z / tau) with z = logit(c); 0 and 1 map to themselves through z = -inf / +inf
__device__ __forceinline__ double sts_sigma(double z, double tau) { return 1.0 / (1.0 + exp(-z / tau)); }

__device__ __forceinline__ double sts_logit(double c) { return log(c) - log1p(-c); }

__device__ __forceinline__ int sts_bin(double p, int M) {
  const int m = (int)floor(p * (double)M);
  return m < M - 1 ? (m > 0 ? m : 0) : M - 1;
}

__global__ void __launch_bounds__(kStsThreads) sts_hist(StsArgs a, int k) {
  extern __shared__ double h[];  // [(J + 1) * M]
  const int HM = (a.J + 1) * a.M;
  for (int i = threadIdx.x; i < HM; i += blockDim.x) h[i] = 0.0;
  __syncthreads();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < a.N; i += stride) {
    double acal = 1.0, araw = 1.0;
    if (k > 0) {
      const double cp = sts_clamp(a.c[i * a.gamma + (k - 1)]);
      acal = a.a_cal[i] * sts_sigma(sts_logit(cp), a.tau[k - 1]);
      araw = a.a_raw[i] * cp;
    }
    a.a_cal[i] = acal;
    a.a_raw[i] = araw;
    const double ck = sts_clamp(a.c[i * a.gamma + k]);
    const double s = a.n[i] >= k + 1 ? 1.0 : 0.0;
    const double pr = araw * ck;
    atomicAdd(&h[a.J * a.M + sts_bin(pr, a.M)], s - pr);
    const double z = sts_logit(ck);
    for (int j = 0; j < a.J; ++j) {
      const double p = acal * sts_sigma(z, __ldg(a.grid + j));
      atomicAdd(&h[j * a.M + sts_bin(p, a.M)], s - p);
    }
  }
  __syncthreads();
  double* hk = a.hist + (size_t)k * HM;
  for (int i = threadIdx.x; i < HM; i += blockDim.x)
    if (h[i] != 0.0) atomicAdd(&hk[i], h[i]);
}

__global__ void __launch_bounds__(kStsThreads) sts_select(StsArgs a, int k) {
  __shared__ double se[kStsThreads / 32];
  __shared__ int sj[kStsThreads / 32];
  const int HM = (a.J + 1) * a.M;
  const double* hk = a.hist + (size_t)k * HM;
  const double invN = 1.0 / (double)a.N;
  double best = DBL_MAX;
  int bj = a.J;
  for (int j = threadIdx.x; j < a.J; j += blockDim.x) {
    double e = 0.0;
    for (int m = 0; m < a.M; ++m) e += fabs(hk[j * a.M + m]);
    e *= invN;
    if (a.curve) a.curve[(size_t)k * a.J + j] = e;
    if (e < best) {  // j ascends: the first minimum of this thread's values
      best = e;
      bj = j;
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
    if (ob < best || (ob == best && oj < bj)) {
      best = ob;
      bj = oj;
    }
  }
  if (lane == 0) {
    se[warp] = best;
    sj[warp] = bj;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kStsThreads / 32; ++w)
      if (se[w] < best || (se[w] == best && sj[w] < bj)) {
        best = se[w];
        bj = sj[w];
      }
    if (bj >= a.J) bj = 0;  // no finite ECE (a temperature <= 0 or NaN in the grid)
    double er = 0.0;
    for (int m = 0; m < a.M; ++m) er += fabs(hk[a.J * a.M + m]);
    a.tau[k] = a.grid[bj];
    if (a.index) a.index[k] = bj;
    if (a.ece_cal) a.ece_cal[k] = best;
    if (a.ece_raw) a.ece_raw[k] = er * invN;
  }
}

__global__ void sts_apply_kernel(const float* c, const double* tau, long long total, int gamma, float* out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int k = (int)(i % gamma);
  out[i] = __double2float_rn(sts_sigma(sts_logit(sts_clamp(c[i])), __ldg(tau + k)));
}

struct StsLayout {
  size_t a_cal, a_raw, hist, total;
};

StsLayout sts_layout(long long N, int gamma, int J, int M) {
  StsLayout L;
  L.a_cal = 0;
  L.a_raw = align_up((size_t)N * 8, 256);
  L.hist = L.a_raw + align_up((size_t)N * 8, 256);
  L.total = L.hist + align_up((size_t)gamma * (J + 1) * M * 8, 256);
  return L;
}

}  // namespace

size_t sts_workspace_bytes(long long N, int gamma, int n_grid, int n_bins) {
  return sts_layout(N, gamma, n_grid, n_bins).total;
}

dspark_status launch_sts_fit(const StsCall& c) {
  const StsLayout Ly = sts_layout(c.N, c.gamma, c.n_grid, c.n_bins);
  uint8_t* ws = static_cast<uint8_t*>(c.ws);
  StsArgs a{};
  a.c = c.c;
  a.n = c.n_acc;
  a.N = c.N;
  a.gamma = c.gamma;
  a.J = c.n_grid;
  a.M = c.n_bins;
  a.grid = c.grid;
  a.a_cal = reinterpret_cast<double*>(ws + Ly.a_cal);
  a.a_raw = reinterpret_cast<double*>(ws + Ly.a_raw);
  a.hist = reinterpret_cast<double*>(ws + Ly.hist);
  a.tau = c.tau;
  a.index = c.index;
  a.ece_raw = c.ece_raw;
  a.ece_cal = c.ece_cal;
  a.curve = c.curve;
  cudaError_t rc = cudaMemsetAsync(a.hist, 0, (size_t)c.gamma * (c.n_grid + 1) * c.n_bins * 8, c.stream);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaMemsetAsync: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  const size_t smem = (size_t)(c.n_grid + 1) * c.n_bins * 8;
  rc = ensure_smem_attr((const void*)sts_hist, smem);
  if (rc != cudaSuccess) {
    set_error(std::string("cudaFuncSetAttribute(sts_hist): ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  // enough CTAs to fill the SMs (a few per SM where shared memory allows), none without samples
  const long long want = (c.N + kStsThreads - 1) / kStsThreads;
  const int per_sm = smem <= 48 * 1024 ? 4 : (smem <= 96 * 1024 ? 2 : 1);
  const int ctas = (int)std::min<long long>(want, (long long)device_sm_count() * per_sm);
  for (int k = 0; k < c.gamma; ++k) {
    sts_hist<<<ctas, kStsThreads, smem, c.stream>>>(a, k);
    sts_select<<<1, kStsThreads, 0, c.stream>>>(a, k);
  }
  rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("sts launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

dspark_status launch_sts_apply(const float* c, const double* tau, int B, int gamma, float* out, cudaStream_t stream) {
  const long long total = (long long)B * gamma;
  const int threads = 256;
  sts_apply_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, stream>>>(c, tau, total, gamma, out);
  const cudaError_t rc = cudaGetLastError();
  if (rc != cudaSuccess) {
    set_error(std::string("sts apply launch: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return DSPARK_OK;
}

}  // namespace dspark
