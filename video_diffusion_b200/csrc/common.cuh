// common.cuh -- shapes, scratch layout and kernel entry declarations shared by
// the translation units of libsolattn.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sol {

// Geometry of one call.  Bq == Bk == B; blocks are contiguous runs of B
// tokens in sequence order and the last one holds n_last = L - (N-1) B tokens.
struct Geometry {
  int bH;      // batch * heads
  int L;       // tokens
  int d;       // head dimension
  int B;       // block size (query and key)
  int N;       // blocks per head, ceil(L / B)
  int W;       // 32-bit words per selection-mask row, ceil(N / 32)
  int nchunk;  // pooled-key chunks of B pooled keys, ceil(N / B)
  int n_last;  // tokens in the last block
  int nitems;  // bH * N work items (one per query block)
};

// Device scratch used by one forward call.
struct Scratch {
  float* qbar;     // [bH, N, d]  mean query per block, fp32
  float* kbar;     // [bH, N, d]  mean key per block, fp32 (routing)
  void* kbar_op;   // [bH, N, d]  mean key per block in the attention kernel's operand type
  void* vbar_op;   // [bH, N, d]  V-hat_j / n_j in the attention kernel's operand type
  uint32_t* mask;  // [bH, N, W]  bit j of row i: key block j selected for query block i
  int32_t* counts; // [bH, N]     |S_i|
  int32_t* tiles;  // [bH, N]     tiles of the attention loop: |S_i| + pooled-key chunks used
  int32_t* order;  // [bH * N]    work items, head-major, heaviest first within a head
  int32_t* work_counter;  // 1 int, zeroed before the attention kernel
};

constexpr int kRouteMaxN = 40960;   // pooled keys per head the router handles
constexpr int kOrderMaxN = 8192;    // query blocks per head the sorter handles

// Prologue launches (prologue.cu).
cudaError_t launch_pool(int in_dtype, int op_dtype, const void* q, const void* k, const void* v,
                        const Geometry& g, const Scratch& s, cudaStream_t st);
cudaError_t launch_route(const Geometry& g, const Scratch& s, float beta, int beta_mode, int correction,
                         cudaStream_t st);
cudaError_t launch_order(const Geometry& g, const Scratch& s, cudaStream_t st);

// Attention launches.
// correction = 0: keep-or-drop (pooled-key tiles skipped, empty rows give 0).
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* out, const Geometry& g,
                           const Scratch& s, cudaStream_t st, uint64_t wait_limit_ns, int correction);
cudaError_t launch_attn_simt(int dtype, const void* q, const void* k, const void* v, void* out,
                             const Geometry& g, const Scratch& s, cudaStream_t st, int correction);
cudaError_t read_device_status(cudaStream_t st, int32_t* word);

}  // namespace sol
