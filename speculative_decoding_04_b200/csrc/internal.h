// Host-side interface between the C ABI (api.cu) and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

#include "../../include/dspark.h"

namespace dspark {

void set_error(const std::string& msg);

struct Options {
  int draft_tc_min_b = 1;        // bf16 drafts with at least this many requests use the tensor-core path
  int draft_force_path = 0;      // 0 auto, 1 CUDA-core GEMV, 2 tensor cores
  int draft_pdl = 1;             // chain the draft kernels with programmatic dependent launch
  int draft_fused = 1;           // tensor-core draft: all steps in one cooperative launch
  int verify_cluster = 0;        // 0 auto, else the cluster size (1, 2, 4, 8, 16)
  int verify_persistent = 1;     // sampled verify / labels: persistent clusters with double-buffered rows (0: one cluster per row)
  int verify_impl = 0;           // verify with a workspace: 0 streaming kernels, 1 column-sliced, 2 per-row
  int verify_groups = 0;         // sliced verify: CTA groups (0: slices of about 16 KB per row)
  int verify_stream_cluster = 0; // CTAs per cluster of the streaming verify (1 to 16; 0: automatic)
  int verify_stream_l2hint = 1;  // streaming verify: first-pass copies evict-last, second-pass evict-first
  int sm_count = 0;              // 0: query the device
  // test-only: make the bounded device waits give up sooner and one of them unsatisfiable, so that
  // a test can check that the kernels return with a timeout status (never on in normal use)
  long debug_wait_limit = 0;      // draft: polls per wait; streaming verify: nanoseconds (0: defaults)
  int debug_unreachable_barrier = 0;  // 1: the draft's first grid barrier; 2: the streaming verify's exchange
};
// A copy of the process-wide options, taken under their lock (dspark_set_option may run on
// another thread).
Options options();

// cudaFuncSetAttribute for the dynamic shared-memory size of `func`, raised as needed and
// remembered per device (a process may drive several GPUs; each needs the attribute once).
cudaError_t ensure_smem_attr(const void* func, size_t bytes);
// Allow cluster sizes above 8 for `func` on the current device (remembered per device).
cudaError_t ensure_nonportable_cluster(const void* func);

int device_sm_count();

struct DraftCall {
  const float* U;
  const void* W1;
  const void* W2;
  int w_dtype;
  const int32_t* x0;
  const float* u_draft;
  int B, gamma, V, r;
  float T;
  int layout;  // of U and ld_out: DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR
  int32_t* x_out;
  float* ld_out;
  uint32_t* flags;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  const void* Wh = nullptr;  // recurrent head: [r][r] state matrix (null: the Markov head)
  float* h_out = nullptr;    // recurrent head: [B][gamma][r] fp32 states, or null
};

struct VerifyCall {
  const float* ld;
  const float* lt;
  const int32_t* x;
  const int32_t* L;
  const float* u_acc;
  const float* u_res;
  int B, gamma, V, lt_rows;
  float T;
  int ld_layout;     // DSPARK_POSITION_MAJOR or DSPARK_REQUEST_MAJOR
  int do_verify;
  int per_row_only;  // 1: the per-row cluster kernels only (their workspace layout), never the streaming ones
  int32_t* n_acc;
  int32_t* y_out;
  float* c_star;
  uint32_t* flags;
  void* ws;
  size_t ws_bytes;
  cudaStream_t stream;
  const int64_t* lt_off = nullptr;  // flattened l_t: request b's rows start at lt_off[b] (nullptr: padded)
  long long lt_nrows = 0;           // rows of the flattened l_t
};

struct StsCall {
  const float* c;
  const int32_t* n_acc;
  long long N;
  int gamma, n_grid, n_bins;
  const double* grid;
  double* tau;
  int32_t* index;
  double* ece_raw;
  double* ece_cal;
  double* curve;
  void* ws;
  cudaStream_t stream;
};
size_t sts_workspace_bytes(long long N, int gamma, int n_grid, int n_bins);
dspark_status launch_sts_fit(const StsCall& c);
dspark_status launch_sts_apply(const float* c, const double* tau, int B, int gamma, float* out, cudaStream_t stream);
constexpr size_t kStsMaxHistBytes = 200 * 1024;  // (n_grid + 1) * n_bins fp64 sums in shared memory

dspark_status launch_ragged_layout(const int32_t* L, int B, int gamma, int64_t* lt_off, int32_t* tags,
                                   cudaStream_t stream);

// State of the asynchronous (t-2) scheduler, DSPARK_T2_RING_BYTES of caller-owned device memory;
// the field offsets are part of the C interface.
struct T2Ring {
  long long t;       // steps taken on this ring
  int D[4];          // D*_s of step s at D[s % 4]
  unsigned tie[4];   // that decision was a near-tie
  double theta[4];   // Θ_s(D*_s)
  int K[4];          // capacity applied at step s
};
static_assert(offsetof(T2Ring, D) == 8 && offsetof(T2Ring, tie) == 24 && offsetof(T2Ring, theta) == 40 &&
                  offsetof(T2Ring, K) == 72 && sizeof(T2Ring) <= DSPARK_T2_RING_BYTES,
              "T2Ring layout");

struct ScheduleCall {
  const float* c;
  const double* sps;
  int B, gamma, D_max, mode;
  int32_t* L_out;
  float* a_out;
  double* theta_out;
  uint32_t* flags;
  cudaStream_t stream;
  T2Ring* ring = nullptr;
  int K_init = -1;
  int32_t* K_out = nullptr;
};

size_t draft_workspace_bytes(int B, int gamma, int V, int r);
size_t rnn_draft_workspace_bytes(int B, int gamma, int V, int r);
size_t verify_workspace_bytes(int B, int gamma, int V);
size_t verify_rows_workspace_bytes(int B, int gamma);

dspark_status launch_draft(const DraftCall& c);
dspark_status launch_verify(const VerifyCall& c);
dspark_status launch_verify_stream(const VerifyCall& c);
size_t stream_verify_workspace_bytes(int B, int gamma, int V);
dspark_status launch_verify_sliced(const VerifyCall& c);
size_t sliced_verify_workspace_bytes(int B, int gamma, int V);
dspark_status launch_schedule(const ScheduleCall& c);

constexpr int kMaxGamma = 64;
constexpr int kMaxScheduleItems = 16384;
constexpr size_t kWsHeader = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Element strides of the l_d (or U) row of position k and request b: row = k * sk + b * sb.
inline void ld_strides(int layout, int B, int gamma, int V, size_t& sk, size_t& sb) {
  if (layout == DSPARK_REQUEST_MAJOR) {
    sk = (size_t)V;
    sb = (size_t)gamma * V;
  } else {
    sk = (size_t)B * V;
    sb = (size_t)V;
  }
}

}  // namespace dspark
