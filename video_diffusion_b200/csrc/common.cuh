// common.cuh -- shapes, scratch layout and kernel entry declarations shared by
// the translation units of libsolattn.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sol {

// Geometry of one call.  Query and key blocks are contiguous runs of Bq and
// Bk tokens in sequence order; the last query block holds nq_last tokens and
// the last key block nk_last.
struct Geometry {
  int bH;       // batch * heads
  int L;        // tokens
  int d;        // head dimension
  int Bq, Bk;   // query / key block size
  int Nq, Nk;   // blocks per head: ceil(L / Bq), ceil(L / Bk)
  int W;        // 32-bit words per selection-mask row, ceil(Nk / 32)
  int nchunk;   // chunks of kChunk pooled keys, ceil(Nk / kChunk)
  int nq_last;  // tokens in the last query block
  int nk_last;  // tokens in the last key block
  int nitems;   // bH * Nq work items (one per query block)
};

// Pooled keys per chunk of the approximate path: one 128-column score tile of
// the tensor-core kernel.
constexpr int kChunk = 128;

// Device scratch used by one forward call.
struct Scratch {
  float* qbar;     // [bH, Nq, d]  mean query per block, fp32
  float* kbar;     // [bH, Nk, d]  mean key per block, fp32 (routing)
  void* kbar_op;   // [bH, Nk, d]  mean key per block in the attention kernel's operand type
  void* vbar_op;   // [bH, Nk, d]  V-hat_j / n_j in the attention kernel's operand type
  float* kvar;     // [bH, d]      Var_j(K-bar_j,c), population (diagonal sigma only)
  uint32_t* mask;  // [bH, Nq, W]  bit j of row i: key block j selected for query block i (may be null)
  float* tau;      // [bH, Nq]     tau_i of Eq. 4
  int32_t* counts; // [bH, Nq]     |S_i|
  int32_t* tiles;  // [bH, Nq]     tiles of the attention loop: |S_i| + pooled-key chunks used
  int32_t* order;  // [bH * Nq]    work items, head-major, heaviest first within a head
  int32_t* work_counter;  // 1 int, zeroed before the attention kernel
  // routing diagnostics (null unless asked for): near[i] = number of key
  // blocks j with |s_ij - tau_i| < near_margin
  int32_t* near;
  float near_margin;
};

constexpr int kMaxSlices = 65535;  // batch * heads: the prologue grids put it in gridDim.y
constexpr int kRouteMaxN = 6144;    // pooled keys per head the router handles (8 score rows in shared memory)
constexpr int kOrderMaxN = 8192;    // query blocks per head the sorter handles

// How sigma_i of Eq. 4 is estimated.
enum SigmaMode : int {
  kSigmaEq5 = 0,       // population std of the proxy-score row (Eq. 5)
  kSigmaDiagonal = 1,  // scale * sqrt(sum_c Q-bar_ic^2 Var_j(K-bar_jc)): the diagonal estimator
};

// Prologue launches (prologue.cu).
cudaError_t launch_pool(int in_dtype, int op_dtype, const void* q, const void* k, const void* v,
                        const Geometry& g, const Scratch& s, cudaStream_t st);
// pair != 0: the attention kernel takes two selected key blocks per tile.
cudaError_t launch_route(const Geometry& g, const Scratch& s, float beta, int beta_mode, int correction,
                         int sigma_mode, int pair, cudaStream_t st);
// Heaviest-first order of the work items of each head; an item is `group`
// consecutive query blocks (1, or 2 for the tensor-core kernel's 64-token
// query blocks).
cudaError_t launch_order(const Geometry& g, const Scratch& s, int group, cudaStream_t st);

// Attention launches.
// correction = 0: keep-or-drop (pooled-key tiles skipped, empty rows give 0).
// route_inkernel != 0: the tensor-core kernel decides S_i itself from s.qbar,
// s.kbar and s.tau (needs W <= 64) and never reads s.mask.
constexpr int kInKernelMaxW = 64;
// test_stall != 0 (failure-detection tests only): the MMA thread of every CTA
// never signals its first S, so the waits on it run out and the kernel takes
// its abort path.
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* out, const Geometry& g,
                           const Scratch& s, cudaStream_t st, uint64_t wait_limit_ns, int correction,
                           int route_inkernel, int test_stall = 0);
cudaError_t launch_attn_simt(int dtype, const void* q, const void* k, const void* v, void* out,
                             const Geometry& g, const Scratch& s, cudaStream_t st, int correction);
cudaError_t read_device_status(cudaStream_t st, int32_t* word);
// Per-CTA record of the last tensor-core attention launch: n rows of
// {start ns, end ns, items, tiles} (rows past the launch's grid are stale).
constexpr int kMaxCtaTimes = 1024;
cudaError_t read_cta_times(cudaStream_t st, unsigned long long* host, int n);
int last_attn_grid();

}  // namespace sol
