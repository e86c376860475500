// C ABI of libdspark.so: host-side argument checks and dispatch to the kernel launchers.
// Every entry point validates its arguments before anything is launched and returns a
// dspark_status; nothing here allocates device memory.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <utility>

#include "internal.h"

namespace dspark {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

static std::mutex g_opt_mu;

static Options& options_ref() {
  static Options o;
  static std::once_flag once;
  std::call_once(once, [] {
    if (const char* e = std::getenv("DSPARK_DRAFT_TC_MIN_B")) o.draft_tc_min_b = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_DRAFT_PATH")) o.draft_force_path = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_DRAFT_PDL")) o.draft_pdl = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_DRAFT_FUSED")) o.draft_fused = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_VERIFY_CLUSTER")) o.verify_cluster = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_VERIFY_PERSISTENT")) o.verify_persistent = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_VERIFY_IMPL")) o.verify_impl = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_VERIFY_GROUPS")) o.verify_groups = std::atoi(e);
    if (const char* e = std::getenv("DSPARK_VERIFY_STREAM_CLUSTER")) o.verify_stream_cluster = std::atoi(e);
  });
  return o;
}

Options options() {
  std::lock_guard<std::mutex> lock(g_opt_mu);
  return options_ref();
}

// (device, function) -> the largest dynamic shared-memory size set so far; a second map for the
// non-portable cluster attribute.
static std::mutex g_attr_mu;
static std::map<std::pair<int, const void*>, size_t> g_smem_attr;
static std::set<std::pair<int, const void*>> g_np_attr;

cudaError_t ensure_smem_attr(const void* func, size_t bytes) {
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  size_t& done = g_smem_attr[{dev, func}];
  if (bytes <= done) return cudaSuccess;
  rc = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (rc == cudaSuccess) done = bytes;
  return rc;
}

cudaError_t ensure_nonportable_cluster(const void* func) {
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  if (g_np_attr.count({dev, func})) return cudaSuccess;
  rc = cudaFuncSetAttribute(func, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (rc == cudaSuccess) g_np_attr.insert({dev, func});
  return rc;
}

int device_sm_count() {
  const int forced = options().sm_count;
  if (forced > 0) return forced;
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

static dspark_status einval(const std::string& msg) {
  set_error(msg);
  return DSPARK_EINVAL;
}

}  // namespace dspark

using namespace dspark;

extern "C" {

const char* dspark_status_string(int status) {
  switch (status) {
    case DSPARK_OK: return "DSPARK_OK";
    case DSPARK_EINVAL: return "DSPARK_EINVAL";
    case DSPARK_ECUDA: return "DSPARK_ECUDA";
    case DSPARK_ENOTIMPL: return "DSPARK_ENOTIMPL";
    case DSPARK_ETIMEOUT: return "DSPARK_ETIMEOUT";
    default: return "DSPARK_UNKNOWN";
  }
}

const char* dspark_last_error(void) { return g_last_error.c_str(); }

int dspark_set_option(const char* key, long value) {
  if (!key) return einval("dspark_set_option: null key");
  std::lock_guard<std::mutex> lock(g_opt_mu);
  Options& o = options_ref();
  if (!std::strcmp(key, "draft_tc_min_b")) o.draft_tc_min_b = (int)value;
  else if (!std::strcmp(key, "draft_path")) o.draft_force_path = (int)value;
  else if (!std::strcmp(key, "draft_pdl")) o.draft_pdl = (int)value;
  else if (!std::strcmp(key, "draft_fused")) o.draft_fused = (int)value;
  else if (!std::strcmp(key, "verify_cluster")) o.verify_cluster = (int)value;
  else if (!std::strcmp(key, "verify_persistent")) o.verify_persistent = (int)value;
  else if (!std::strcmp(key, "verify_impl")) o.verify_impl = (int)value;
  else if (!std::strcmp(key, "verify_groups")) o.verify_groups = (int)value;
  else if (!std::strcmp(key, "verify_stream_cluster")) o.verify_stream_cluster = (int)value;
  else if (!std::strcmp(key, "verify_stream_l2hint")) o.verify_stream_l2hint = (int)value;
  else if (!std::strcmp(key, "sm_count")) o.sm_count = (int)value;
  else if (!std::strcmp(key, "debug_wait_limit")) o.debug_wait_limit = value;
  else if (!std::strcmp(key, "debug_unreachable_barrier")) o.debug_unreachable_barrier = (int)value;
  else return einval(std::string("dspark_set_option: unknown key ") + key);
  return DSPARK_OK;
}

size_t dspark_workspace_size(int which, int B, int gamma, int V, int r) {
  if (B <= 0 || gamma <= 0 || V <= 0) return 0;
  switch (which) {
    case DSPARK_WS_DRAFT: return draft_workspace_bytes(B, gamma, V, r);
    case DSPARK_WS_VERIFY: return verify_workspace_bytes(B, gamma, V);
    case DSPARK_WS_SCHEDULE: return 0;
    case DSPARK_WS_RNN_DRAFT: return rnn_draft_workspace_bytes(B, gamma, V, r);
    default: return 0;
  }
}

int dspark_workspace_status(const void* ws, void* stream) {
  if (!ws) return einval("dspark_workspace_status: null workspace");
  uint32_t st = 0;
  cudaError_t rc = cudaMemcpyAsync(&st, ws, sizeof(st), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (rc == cudaSuccess) rc = cudaStreamSynchronize((cudaStream_t)stream);
  if (rc != cudaSuccess) {
    set_error(std::string("dspark_workspace_status: ") + cudaGetErrorString(rc));
    return DSPARK_ECUDA;
  }
  return st ? DSPARK_ETIMEOUT : DSPARK_OK;
}

int dspark_markov_draft(const float* U, const void* W1, const void* W2, int w_dtype, const int32_t* x0,
                        const float* u_draft, int B, int gamma, int V, int r, float T, int layout, int32_t* x_out,
                        float* ld_out, uint32_t* flags, void* ws, size_t ws_bytes, void* stream) {
  if (!U || !W1 || !W2 || !x0 || !x_out || !ld_out || !flags || !ws) return einval("dspark_markov_draft: null pointer");
  if (T != 0.f && !u_draft) return einval("dspark_markov_draft: u_draft is required when T > 0");
  if (B <= 0 || V < 2 || r <= 0) return einval("dspark_markov_draft: B, r must be >= 1 and V >= 2");
  if (gamma < 1 || gamma > kMaxGamma) return einval("dspark_markov_draft: gamma must be in [1, 64]");
  if (!(T >= 0.f) || std::isinf(T)) return einval("dspark_markov_draft: T must be finite and >= 0");
  if (w_dtype != DSPARK_BF16 && w_dtype != DSPARK_F32) return einval("dspark_markov_draft: w_dtype must be DSPARK_BF16 or DSPARK_F32");
  if (layout != DSPARK_POSITION_MAJOR && layout != DSPARK_REQUEST_MAJOR)
    return einval("dspark_markov_draft: layout must be DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR");
  if ((long long)B * gamma * V >= (1ll << 40)) return einval("dspark_markov_draft: tensor too large");
  if (ws_bytes < draft_workspace_bytes(B, gamma, V, r)) return einval("dspark_markov_draft: workspace too small");
  if ((uintptr_t)ws % 256) return einval("dspark_markov_draft: workspace must be 256-byte aligned");
  DraftCall c{U, W1, W2, w_dtype, x0, u_draft, B, gamma, V, r, T, layout, x_out, ld_out, flags, ws, ws_bytes,
              (cudaStream_t)stream};
  return launch_draft(c);
}

int dspark_rnn_draft(const float* U, const void* W1, const void* W2, const void* Wh, int w_dtype, const int32_t* x0,
                     const float* u_draft, int B, int gamma, int V, int r, float T, int layout, int32_t* x_out,
                     float* ld_out, float* h_out, uint32_t* flags, void* ws, size_t ws_bytes, void* stream) {
  if (!U || !W1 || !W2 || !Wh || !x0 || !x_out || !ld_out || !flags || !ws) return einval("dspark_rnn_draft: null pointer");
  if (T != 0.f && !u_draft) return einval("dspark_rnn_draft: u_draft is required when T > 0");
  if (B <= 0 || V < 2 || r <= 0) return einval("dspark_rnn_draft: B, r must be >= 1 and V >= 2");
  if (r > 1024) return einval("dspark_rnn_draft: r must be <= 1024");
  if (gamma < 1 || gamma > kMaxGamma) return einval("dspark_rnn_draft: gamma must be in [1, 64]");
  if (!(T >= 0.f) || std::isinf(T)) return einval("dspark_rnn_draft: T must be finite and >= 0");
  if (w_dtype != DSPARK_BF16 && w_dtype != DSPARK_F32) return einval("dspark_rnn_draft: w_dtype must be DSPARK_BF16 or DSPARK_F32");
  if (layout != DSPARK_POSITION_MAJOR && layout != DSPARK_REQUEST_MAJOR)
    return einval("dspark_rnn_draft: layout must be DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR");
  if ((long long)B * gamma * V >= (1ll << 40)) return einval("dspark_rnn_draft: tensor too large");
  if (ws_bytes < rnn_draft_workspace_bytes(B, gamma, V, r)) return einval("dspark_rnn_draft: workspace too small");
  if ((uintptr_t)ws % 256) return einval("dspark_rnn_draft: workspace must be 256-byte aligned");
  DraftCall c{U, W1, W2, w_dtype, x0, u_draft, B, gamma, V, r, T, layout, x_out, ld_out, flags, ws, ws_bytes,
              (cudaStream_t)stream};
  c.Wh = Wh;
  c.h_out = h_out;
  return launch_draft(c);
}

int dspark_verify(const float* ld, const float* lt, const int32_t* x, const int32_t* L, const float* u_acc,
                  const float* u_res, int B, int gamma, int V, float T, int ld_layout, int32_t* n_acc, int32_t* y_out,
                  float* c_star, uint32_t* flags, void* ws, size_t ws_bytes, void* stream) {
  if (!ld || !lt || !x || !n_acc || !y_out || !flags || !ws) return einval("dspark_verify: null pointer");
  if (T != 0.f && (!u_acc || !u_res)) return einval("dspark_verify: u_acc and u_res are required when T > 0");
  if (B <= 0 || V < 2) return einval("dspark_verify: B must be >= 1 and V >= 2");
  if (gamma < 1 || gamma > kMaxGamma) return einval("dspark_verify: gamma must be in [1, 64]");
  if (!(T >= 0.f) || std::isinf(T)) return einval("dspark_verify: T must be finite and >= 0");
  if (ld_layout != DSPARK_POSITION_MAJOR && ld_layout != DSPARK_REQUEST_MAJOR)
    return einval("dspark_verify: ld_layout must be DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR");
  if (ws_bytes < verify_workspace_bytes(B, gamma, V)) return einval("dspark_verify: workspace too small");
  if ((uintptr_t)ws % 256) return einval("dspark_verify: workspace must be 256-byte aligned");
  VerifyCall c{ld, lt, x, L, u_acc, u_res, B, gamma, V, gamma + 1, T, ld_layout, 1, 0, n_acc, y_out, c_star, flags, ws, ws_bytes,
               (cudaStream_t)stream};
  return launch_verify(c);
}

int dspark_ragged_layout(const int32_t* L, int B, int gamma, int64_t* lt_off, int32_t* tags, void* stream) {
  if (!L || !lt_off) return einval("dspark_ragged_layout: null pointer");
  if (B <= 0 || gamma < 1 || gamma > kMaxGamma) return einval("dspark_ragged_layout: B >= 1, gamma in [1, 64]");
  return launch_ragged_layout(L, B, gamma, lt_off, tags, (cudaStream_t)stream);
}

int dspark_verify_ragged(const float* ld, const float* lt, const int64_t* lt_off, int64_t lt_nrows, const int32_t* x,
                         const int32_t* L, const float* u_acc, const float* u_res, int B, int gamma, int V, float T,
                         int ld_layout, int32_t* n_acc, int32_t* y_out, float* c_star, uint32_t* flags, void* ws,
                         size_t ws_bytes, void* stream) {
  if (!ld || !lt || !lt_off || !x || !L || !n_acc || !y_out || !flags || !ws)
    return einval("dspark_verify_ragged: null pointer");
  if (T != 0.f && (!u_acc || !u_res)) return einval("dspark_verify_ragged: u_acc and u_res are required when T > 0");
  if (B <= 0 || V < 2) return einval("dspark_verify_ragged: B must be >= 1 and V >= 2");
  if (gamma < 1 || gamma > kMaxGamma) return einval("dspark_verify_ragged: gamma must be in [1, 64]");
  if (lt_nrows < 1) return einval("dspark_verify_ragged: lt_nrows must be >= 1");
  if (!(T >= 0.f) || std::isinf(T)) return einval("dspark_verify_ragged: T must be finite and >= 0");
  if (ld_layout != DSPARK_POSITION_MAJOR && ld_layout != DSPARK_REQUEST_MAJOR)
    return einval("dspark_verify_ragged: ld_layout must be DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR");
  if (ws_bytes < verify_workspace_bytes(B, gamma, V)) return einval("dspark_verify_ragged: workspace too small");
  if ((uintptr_t)ws % 256) return einval("dspark_verify_ragged: workspace must be 256-byte aligned");
  VerifyCall c{ld, lt, x, L, u_acc, u_res, B, gamma, V, gamma + 1, T, ld_layout, 1, 0, n_acc, y_out, c_star, flags, ws, ws_bytes,
               (cudaStream_t)stream};
  c.lt_off = lt_off;
  c.lt_nrows = (long long)lt_nrows;
  return launch_verify(c);
}

size_t dspark_sts_workspace_size(int64_t N, int gamma, int n_grid, int n_bins) {
  if (N < 1 || gamma < 1 || n_grid < 1 || n_bins < 1) return 0;
  return sts_workspace_bytes((long long)N, gamma, n_grid, n_bins);
}

int dspark_sts_fit(const float* c, const int32_t* n_acc, int64_t N, int gamma, const double* grid, int n_grid,
                   int n_bins, double* tau_out, int32_t* index_out, double* ece_raw, double* ece_cal,
                   double* curve_out, void* ws, size_t ws_bytes, void* stream) {
  if (!c || !n_acc || !grid || !tau_out || !ws) return einval("dspark_sts_fit: null pointer");
  if (N < 1 || gamma < 1 || gamma > kMaxGamma) return einval("dspark_sts_fit: N >= 1, gamma in [1, 64]");
  if (n_grid < 1 || n_bins < 1) return einval("dspark_sts_fit: n_grid and n_bins must be >= 1");
  if ((size_t)(n_grid + 1) * (size_t)n_bins * 8 > kStsMaxHistBytes)
    return einval("dspark_sts_fit: (n_grid + 1) * n_bins must be <= 25600");
  if (ws_bytes < sts_workspace_bytes((long long)N, gamma, n_grid, n_bins)) return einval("dspark_sts_fit: workspace too small");
  if ((uintptr_t)ws % 256) return einval("dspark_sts_fit: workspace must be 256-byte aligned");
  StsCall sc{c, n_acc, (long long)N, gamma, n_grid, n_bins, grid, tau_out, index_out, ece_raw, ece_cal, curve_out, ws,
             (cudaStream_t)stream};
  return launch_sts_fit(sc);
}

int dspark_sts_apply(const float* c, const double* tau, int B, int gamma, float* c_out, void* stream) {
  if (!c || !tau || !c_out) return einval("dspark_sts_apply: null pointer");
  if (B < 1 || gamma < 1 || gamma > kMaxGamma) return einval("dspark_sts_apply: B >= 1, gamma in [1, 64]");
  return launch_sts_apply(c, tau, B, gamma, c_out, (cudaStream_t)stream);
}

int dspark_tv_labels(const float* ld, const float* lt, int B, int gamma, int V, int lt_rows, float T, int ld_layout,
                     float* c_star, void* stream) {
  if (!ld || !lt || !c_star) return einval("dspark_tv_labels: null pointer");
  if (B <= 0 || V < 2) return einval("dspark_tv_labels: B must be >= 1 and V >= 2");
  if (gamma < 1 || gamma > kMaxGamma) return einval("dspark_tv_labels: gamma must be in [1, 64]");
  if (lt_rows != gamma && lt_rows != gamma + 1) return einval("dspark_tv_labels: lt_rows must be gamma or gamma+1");
  if (ld_layout != DSPARK_POSITION_MAJOR && ld_layout != DSPARK_REQUEST_MAJOR)
    return einval("dspark_tv_labels: ld_layout must be DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR");
  if (!(T >= 0.f) || std::isinf(T)) return einval("dspark_tv_labels: T must be finite and >= 0");
  VerifyCall c{ld, lt, nullptr, nullptr, nullptr, nullptr, B, gamma, V, lt_rows, T, ld_layout, 0, 0, nullptr, nullptr, c_star,
               nullptr, nullptr, 0, (cudaStream_t)stream};
  return launch_verify(c);
}

int dspark_prefix_schedule(const float* c, const double* sps, int B, int gamma, int D_max, int mode, int32_t* L_out,
                           float* a_out, double* theta_out, uint32_t* flags, void* ws, size_t ws_bytes,
                           void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (!c || !sps || !L_out || !theta_out) return einval("dspark_prefix_schedule: null pointer");
  if (B <= 0 || gamma < 1 || gamma > kMaxGamma) return einval("dspark_prefix_schedule: B >= 1, gamma in [1, 64]");
  if ((long long)B * gamma > kMaxScheduleItems) return einval("dspark_prefix_schedule: B*gamma must be <= 16384");
  if (D_max < 0 || D_max > B * gamma) return einval("dspark_prefix_schedule: D_max must be in [0, B*gamma]");
  if (mode != DSPARK_SCHED_ARGMAX && mode != DSPARK_SCHED_EARLY_STOP) return einval("dspark_prefix_schedule: bad mode");
  ScheduleCall s{c, sps, B, gamma, D_max, mode, L_out, a_out, theta_out, flags, (cudaStream_t)stream};
  return launch_schedule(s);
}

int dspark_prefix_schedule_t2(const float* c, const double* sps, int B, int gamma, int D_max, int mode, int K_init,
                              void* ring, int32_t* L_out, float* a_out, double* theta_out, int32_t* K_out,
                              uint32_t* flags, void* stream) {
  if (!c || !sps || !L_out || !theta_out || !ring) return einval("dspark_prefix_schedule_t2: null pointer");
  if ((uintptr_t)ring % 8 != 0) return einval("dspark_prefix_schedule_t2: ring must be 8-byte aligned");
  if (B <= 0 || gamma < 1 || gamma > kMaxGamma) return einval("dspark_prefix_schedule_t2: B >= 1, gamma in [1, 64]");
  if ((long long)B * gamma > kMaxScheduleItems) return einval("dspark_prefix_schedule_t2: B*gamma must be <= 16384");
  if (D_max < 0 || D_max > B * gamma) return einval("dspark_prefix_schedule_t2: D_max must be in [0, B*gamma]");
  if (mode != DSPARK_SCHED_ARGMAX && mode != DSPARK_SCHED_EARLY_STOP)
    return einval("dspark_prefix_schedule_t2: bad mode");
  ScheduleCall s{c, sps, B, gamma, D_max, mode, L_out, a_out, theta_out, flags, (cudaStream_t)stream};
  s.ring = static_cast<T2Ring*>(ring);
  s.K_init = K_init;
  s.K_out = K_out;
  return launch_schedule(s);
}

}  // extern "C"
