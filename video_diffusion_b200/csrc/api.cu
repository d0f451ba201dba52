// api.cu -- the C ABI of libsolattn (declared in include/sol_attn.h).
//
// Host-side work only: argument checks, scratch carving (one stream-ordered
// allocation per call from a library-owned memory pool that keeps its memory
// between calls), and the launch sequence pool -> route -> order -> attention
// on the caller's stream.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "../../include/sol_attn.h"
#include "common.cuh"

namespace {

using sol::Geometry;
using sol::Scratch;

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s per bounded wait

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_args(const void* q, const void* k, const void* v_or_dummy, const void* out_or_dummy, int batch,
               int heads, int L, int d, int Bq, int Bk, float beta, Geometry* g) {
  if (!q || !k || !v_or_dummy || !out_or_dummy) return SOL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v_or_dummy) || !aligned16(out_or_dummy))
    return SOL_ERR_INVALID_ARG;
  if (batch < 1 || heads < 1 || L < 1 || d < 1 || Bq < 1 || Bk < 1) return SOL_ERR_INVALID_ARG;
  if (std::isnan(beta)) return SOL_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SOL_ERR_UNSUPPORTED;
  if ((Bq != 64 && Bq != 128) || (Bk != 64 && Bk != 128)) return SOL_ERR_UNSUPPORTED;
  const int64_t bH = (int64_t)batch * heads;
  // batch * heads is the y dimension of the prologue kernels' grids
  if (bH > sol::kMaxSlices || bH * (int64_t)L * d >= (int64_t(1) << 40)) return SOL_ERR_UNSUPPORTED;
  const int Nq = (L + Bq - 1) / Bq;
  const int Nk = (L + Bk - 1) / Bk;
  if (Nk > sol::kRouteMaxN) return SOL_ERR_UNSUPPORTED;
  if (bH * Nq >= (int64_t(1) << 31) || bH * Nk >= (int64_t(1) << 31)) return SOL_ERR_UNSUPPORTED;
  g->bH = (int)bH;
  g->L = L;
  g->d = d;
  g->Bq = Bq;
  g->Bk = Bk;
  g->Nq = Nq;
  g->Nk = Nk;
  g->W = (Nk + 31) / 32;
  g->nchunk = (Nk + sol::kChunk - 1) / sol::kChunk;
  g->nq_last = L - (Nq - 1) * Bq;
  g->nk_last = L - (Nk - 1) * Bk;
  g->nitems = (int)(bH * Nq);
  return SOL_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Carves the scratch out of one allocation; returns its size when base is null.
size_t carve(const Geometry& g, size_t op_elem, char* base, Scratch* s) {
  const size_t qpooled = (size_t)g.bH * g.Nq * g.d;
  const size_t kpooled = (size_t)g.bH * g.Nk * g.d;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  s->qbar = reinterpret_cast<float*>(take(qpooled * sizeof(float)));
  s->kbar = reinterpret_cast<float*>(take(kpooled * sizeof(float)));
  s->kbar_op = take(kpooled * op_elem);
  s->vbar_op = take(kpooled * op_elem);
  s->kvar = reinterpret_cast<float*>(take((size_t)g.bH * g.d * sizeof(float)));
  s->mask = reinterpret_cast<uint32_t*>(take((size_t)g.nitems * g.W * sizeof(uint32_t)));
  s->tau = reinterpret_cast<float*>(take((size_t)g.nitems * sizeof(float)));
  s->counts = reinterpret_cast<int32_t*>(take((size_t)g.nitems * sizeof(int32_t)));
  s->tiles = reinterpret_cast<int32_t*>(take((size_t)g.nitems * sizeof(int32_t)));
  s->order = reinterpret_cast<int32_t*>(take((size_t)g.nitems * sizeof(int32_t)));
  s->work_counter = reinterpret_cast<int32_t*>(take(sizeof(int32_t)));
  s->near = nullptr;
  s->near_margin = 0.f;
  return off;
}

// One stream-ordered pool per device for the per-call scratch.  Its release
// threshold is unlimited, so memory freed by one call is reused by the next
// without going back to the driver (the process's default pool is left as
// the application configured it).
constexpr int kPoolDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kPoolDevices] = {};

cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kPoolDevices) return cudaErrorInvalidDevice;
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> lock(g_pool_mu);
    if (!g_pool[dev]) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      e = cudaMemPoolCreate(&g_pool[dev], &props);
      if (e != cudaSuccess) return e;
      uint64_t keep = ~0ull;
      e = cudaMemPoolSetAttribute(g_pool[dev], cudaMemPoolAttrReleaseThreshold, &keep);
      if (e != cudaSuccess) return e;
    }
    pool = g_pool[dev];
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, st);
}

// The tensor-core kernel is built for bf16 with d in {64, 128}, query blocks
// of 128 or 64 tokens (two 64-token blocks share a 128-row tile) and key
// blocks of 128 or 64 (two 64-token blocks share a tile).
bool uses_tensor_cores(int dtype, const Geometry& g) {
  return dtype == SOL_DTYPE_BF16 && (g.d == 128 || g.d == 64) && (g.Bq == 128 || g.Bq == 64) &&
         (g.Bk == 128 || g.Bk == 64);
}

// In-kernel routing runs on the tensor-core kernel with 128-token query
// blocks and at most 64 mask words per row.
bool inkernel_supported(int dtype, const Geometry& g) {
  return uses_tensor_cores(dtype, g) && g.Bq == 128 && g.W <= sol::kInKernelMaxW;
}

// Query blocks per work item of the attention kernel: the tensor-core kernel
// takes 64-token query blocks two at a time (one 128-row tile).
int order_group(bool use_tc, const Geometry& g) { return use_tc && g.Bq == 64 ? 2 : 1; }

int pair_tiles(bool use_tc, const Geometry& g) { return use_tc && g.Bk == 64 ? 1 : 0; }

int beta_mode_of(float beta) { return std::isinf(beta) ? (beta < 0 ? -1 : 1) : 0; }

uint64_t wait_limit_ns() {
  // test hook: a shorter limit makes an expiring wait quick to observe
  const char* e = std::getenv("SOL_ATTN_WAIT_LIMIT_NS");
  if (e && *e) {
    const unsigned long long v = std::strtoull(e, nullptr, 10);
    if (v > 0) return v;
  }
  return kDefaultWaitLimitNs;
}

// Failure-detection test hook: SOL_ATTN_TEST_STALL=1 makes the tensor-core
// kernel's first wait in every CTA unsatisfiable, so that (with a short
// SOL_ATTN_WAIT_LIMIT_NS) the bounded wait runs out and the kernel reports
// SOL_ERR_DEVICE_TIMEOUT through sol_attn_device_status instead of hanging.
int test_stall() {
  const char* e = std::getenv("SOL_ATTN_TEST_STALL");
  return (e && *e && *e != '0') ? 1 : 0;
}

int record(void* const* events, int i, cudaStream_t st) {
  if (!events || !events[i]) return SOL_OK;
  return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess ? SOL_OK : SOL_ERR_CUDA;
}

int forward_impl(const void* q, const void* k, const void* v, void* out, int dtype, int batch, int heads, int L,
                 int d, int Bq, int Bk, float beta, unsigned flags, void* const* events, cudaStream_t st) {
  if (dtype != SOL_DTYPE_BF16 && dtype != SOL_DTYPE_F32) return SOL_ERR_INVALID_ARG;
  if (flags & ~(SOL_FLAG_KEEP_OR_DROP | SOL_FLAG_DIAGONAL_SIGMA | SOL_FLAG_ROUTE_IN_KERNEL))
    return SOL_ERR_INVALID_ARG;
  const int correction = (flags & SOL_FLAG_KEEP_OR_DROP) ? 0 : 1;
  const int sigma_mode = (flags & SOL_FLAG_DIAGONAL_SIGMA) ? sol::kSigmaDiagonal : sol::kSigmaEq5;
  const int inkernel = (flags & SOL_FLAG_ROUTE_IN_KERNEL) ? 1 : 0;
  Geometry g;
  int rc = check_args(q, k, v, out, batch, heads, L, d, Bq, Bk, beta, &g);
  if (rc != SOL_OK) return rc;
  const bool use_tc = uses_tensor_cores(dtype, g);
  if (inkernel && !inkernel_supported(dtype, g)) return SOL_ERR_UNSUPPORTED;
  const int op_dtype = use_tc ? 0 : 1;  // operand type of K-bar / V-bar: bf16 for tensor cores
  Scratch s;
  const size_t bytes = carve(g, use_tc ? 2 : 4, nullptr, &s);
  void* base = nullptr;
  if (scratch_alloc(&base, bytes, st) != cudaSuccess) {
    cudaGetLastError();
    return SOL_ERR_NO_MEMORY;
  }
  carve(g, use_tc ? 2 : 4, static_cast<char*>(base), &s);
  if (inkernel) s.mask = nullptr;  // no decision record: the attention kernel decides
  cudaError_t e = cudaSuccess;
  const int in_dtype = dtype == SOL_DTYPE_BF16 ? 0 : 1;
  if ((rc = record(events, 0, st)) != SOL_OK) goto done;
  e = sol::launch_pool(in_dtype, op_dtype, q, k, v, g, s, st);
  if (e != cudaSuccess) goto done;
  if ((rc = record(events, 1, st)) != SOL_OK) goto done;
  e = sol::launch_route(g, s, beta, beta_mode_of(beta), correction, sigma_mode, pair_tiles(use_tc, g), st);
  if (e != cudaSuccess) goto done;
  e = sol::launch_order(g, s, order_group(use_tc, g), st);
  if (e != cudaSuccess) goto done;
  if ((rc = record(events, 2, st)) != SOL_OK) goto done;
  if (use_tc) {
    e = cudaMemsetAsync(s.work_counter, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) goto done;
    e = sol::launch_attn_tc(q, k, v, out, g, s, st, wait_limit_ns(), correction, inkernel, test_stall());
  } else {
    e = sol::launch_attn_simt(in_dtype, q, k, v, out, g, s, st, correction);
  }
  if (e != cudaSuccess) goto done;
  rc = record(events, 3, st);
done:
  cudaFreeAsync(base, st);
  if (e != cudaSuccess) return SOL_ERR_CUDA;
  return rc;
}

}  // namespace

extern "C" {

int sol_attn_forward(const void* q, const void* k, const void* v, void* out, int batch, int heads, int L, int d,
                     int Bq, int Bk, float beta, void* stream) {
  return forward_impl(q, k, v, out, SOL_DTYPE_BF16, batch, heads, L, d, Bq, Bk, beta, 0u, nullptr,
                      static_cast<cudaStream_t>(stream));
}

int sol_attn_forward_f32(const float* q, const float* k, const float* v, float* out, int batch, int heads, int L,
                         int d, int Bq, int Bk, float beta, void* stream) {
  return forward_impl(q, k, v, out, SOL_DTYPE_F32, batch, heads, L, d, Bq, Bk, beta, 0u, nullptr,
                      static_cast<cudaStream_t>(stream));
}

int sol_attn_forward_ex(const void* q, const void* k, const void* v, void* out, int dtype, int batch, int heads,
                        int L, int d, int Bq, int Bk, float beta, unsigned int flags, void* const* events,
                        void* stream) {
  return forward_impl(q, k, v, out, dtype, batch, heads, L, d, Bq, Bk, beta, flags, events,
                      static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Pooling and routing only (the forward's kernels, run the same way): counts
// (and optionally the mask, or the near-tie counts) of every query block.
int stats_impl(const void* q, const void* k, int32_t* counts, uint32_t* mask_or_null, int32_t* near,
               float near_margin, int batch, int heads, int L, int d, int Bq, int Bk, float beta, int dtype,
               unsigned int flags, void* stream) {
  if (dtype != SOL_DTYPE_BF16 && dtype != SOL_DTYPE_F32) return SOL_ERR_INVALID_ARG;
  if (flags & ~SOL_FLAG_DIAGONAL_SIGMA) return SOL_ERR_INVALID_ARG;
  const int sigma_mode = (flags & SOL_FLAG_DIAGONAL_SIGMA) ? sol::kSigmaDiagonal : sol::kSigmaEq5;
  Geometry g;
  int rc = check_args(q, k, q, q, batch, heads, L, d, Bq, Bk, beta, &g);
  if (rc != SOL_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch s;
  const size_t bytes = carve(g, 4, nullptr, &s);
  void* base = nullptr;
  if (scratch_alloc(&base, bytes, st) != cudaSuccess) {
    cudaGetLastError();
    return SOL_ERR_NO_MEMORY;
  }
  carve(g, 4, static_cast<char*>(base), &s);
  if (counts) s.counts = counts;
  if (mask_or_null) s.mask = mask_or_null;
  s.near = near;
  s.near_margin = near_margin;
  s.kbar_op = nullptr;  // routing needs the fp32 pooled vectors only
  cudaError_t e = sol::launch_pool(dtype == SOL_DTYPE_BF16 ? 0 : 1, 1, q, k, nullptr, g, s, st);
  if (e == cudaSuccess) e = sol::launch_route(g, s, beta, beta_mode_of(beta), 1, sigma_mode, 0, st);
  cudaFreeAsync(base, st);
  return e == cudaSuccess ? SOL_OK : SOL_ERR_CUDA;
}

}  // namespace

extern "C" {

int sol_attn_stats_ex(const void* q, const void* k, int32_t* counts, uint32_t* mask_or_null, int batch, int heads,
                      int L, int d, int Bq, int Bk, float beta, int dtype, unsigned int flags, void* stream) {
  if (!counts) return SOL_ERR_INVALID_ARG;
  return stats_impl(q, k, counts, mask_or_null, nullptr, 0.f, batch, heads, L, d, Bq, Bk, beta, dtype, flags,
                    stream);
}

int sol_attn_near_ties(const void* q, const void* k, int32_t* near_ties, float margin, int batch, int heads,
                       int L, int d, int Bq, int Bk, float beta, int dtype, unsigned int flags, void* stream) {
  if (!near_ties || !(margin >= 0.f) || std::isinf(margin)) return SOL_ERR_INVALID_ARG;
  return stats_impl(q, k, nullptr, nullptr, near_ties, margin, batch, heads, L, d, Bq, Bk, beta, dtype, flags,
                    stream);
}

int sol_attn_stats(const void* q, const void* k, int32_t* counts, uint32_t* mask_or_null, int batch, int heads,
                   int L, int d, int Bq, int Bk, float beta, int dtype, void* stream) {
  return sol_attn_stats_ex(q, k, counts, mask_or_null, batch, heads, L, d, Bq, Bk, beta, dtype, 0u, stream);
}

int sol_attn_device_status(void* stream, int32_t* detail) {
  int32_t w = 0;
  if (sol::read_device_status(static_cast<cudaStream_t>(stream), &w) != cudaSuccess) return SOL_ERR_CUDA;
  if (detail) *detail = w;
  return w == 0 ? SOL_OK : SOL_ERR_DEVICE_TIMEOUT;
}

int sol_attn_cta_times(void* stream, uint64_t* rows, int max_rows) {
  if (!rows || max_rows < 0) return SOL_ERR_INVALID_ARG;
  int n = sol::last_attn_grid();
  if (n > max_rows) n = max_rows;
  if (n > sol::kMaxCtaTimes) n = sol::kMaxCtaTimes;
  if (n == 0) return 0;
  if (sol::read_cta_times(static_cast<cudaStream_t>(stream), reinterpret_cast<unsigned long long*>(rows), n) !=
      cudaSuccess)
    return SOL_ERR_CUDA;
  return n;
}

const char* sol_attn_status_string(int status) {
  switch (status) {
    case SOL_OK: return "SOL_OK";
    case SOL_ERR_INVALID_ARG: return "SOL_ERR_INVALID_ARG";
    case SOL_ERR_UNSUPPORTED: return "SOL_ERR_UNSUPPORTED";
    case SOL_ERR_CUDA: return "SOL_ERR_CUDA";
    case SOL_ERR_NO_MEMORY: return "SOL_ERR_NO_MEMORY";
    case SOL_ERR_DEVICE_TIMEOUT: return "SOL_ERR_DEVICE_TIMEOUT";
    default: return "SOL_ERR_UNKNOWN";
  }
}

int sol_attn_version(void) { return 105; }

}  // extern "C"

// ----------------------------------------------------------------------------- forward without allocation
//
// Some callers cannot let a library allocate device memory: runtimes that load
// this code as a plugin and hand out every byte of device memory themselves,
// and serving loops that reserve all memory up front and treat any further
// allocation (which can block, fail under fragmentation, or take memory meant
// for activations) as an error.  sol_attn_forward_noalloc serves them with the
// same kernels as sol_attn_forward, taking its scratch from the fixed array
// below instead of a stream-ordered allocation.

namespace {

// Fixed scratch, reserved on every GPU that loads this library until the
// process exits.  At Bk = 128, 48 MiB holds the scratch of the Wan2.1 720p
// call (40 heads, L = 75600: about 37 MiB) and of the HunyuanVideo 720p call
// (about 36 MiB); with Bk = 64 those calls need about 61 and 60 MiB and are
// refused with SOL_ERR_NO_MEMORY.
constexpr size_t kNoAllocScratchBytes = size_t(48) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the symbol; the address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SOL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SOL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return SOL_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SOL_OK;
}

}  // namespace

extern "C" int sol_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out, int batch,
                                        int heads, int L, int d, int Bq, int Bk, float beta, void* stream) {
  Geometry g;
  int rc = check_args(q, k, v, out, batch, heads, L, d, Bq, Bk, beta, &g);
  if (rc != SOL_OK) return rc;
  const bool use_tc = uses_tensor_cores(SOL_DTYPE_BF16, g);
  const int op_dtype = use_tc ? 0 : 1;
  Scratch s;
  const size_t bytes = carve(g, use_tc ? 2 : 4, nullptr, &s);
  if (bytes > kNoAllocScratchBytes) return SOL_ERR_NO_MEMORY;  // call too large for the fixed scratch
  void* base = nullptr;
  if ((rc = noalloc_scratch(&base)) != SOL_OK) return rc;
  carve(g, use_tc ? 2 : 4, static_cast<char*>(base), &s);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Everything the kernels read is rewritten by this call except the work
  // counter, which must start at zero.
  cudaError_t e = sol::launch_pool(0, op_dtype, q, k, v, g, s, st);
  if (e == cudaSuccess)
    e = sol::launch_route(g, s, beta, beta_mode_of(beta), 1, sol::kSigmaEq5, pair_tiles(use_tc, g), st);
  if (e == cudaSuccess) e = sol::launch_order(g, s, order_group(use_tc, g), st);
  if (use_tc) {
    if (e == cudaSuccess) e = cudaMemsetAsync(s.work_counter, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = sol::launch_attn_tc(q, k, v, out, g, s, st, wait_limit_ns(), 1, 0);
  } else if (e == cudaSuccess) {
    e = sol::launch_attn_simt(0, q, k, v, out, g, s, st, 1);
  }
  return e == cudaSuccess ? SOL_OK : SOL_ERR_CUDA;
}

// ----------------------------------------------------------------------------- forward from host memory
//
// sol_attn_forward_host takes q, k, v and out in host memory.  The (batch,
// head) slices are independent all the way through (pooling, routing and the
// attention of one slice read nothing of another), so the call cuts them into
// groups and pipelines the groups through two device staging buffers: while
// group c is computed on the caller's stream, group c + 1's inputs are copied
// in on one internal stream and group c - 1's output is copied back on
// another.  Copy engines and SMs then work at the same time, and the call
// takes about as long as its host-to-device copies.

namespace {

struct HostStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
};
std::mutex g_host_mu;
HostStreams g_host_streams[kMaxDevices];

int host_streams(HostStreams* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SOL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SOL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostStreams& hs = g_host_streams[dev];
  if (!hs.h2d && cudaStreamCreateWithFlags(&hs.h2d, cudaStreamNonBlocking) != cudaSuccess) return SOL_ERR_CUDA;
  if (!hs.d2h && cudaStreamCreateWithFlags(&hs.d2h, cudaStreamNonBlocking) != cudaSuccess) return SOL_ERR_CUDA;
  *out = hs;
  return SOL_OK;
}

constexpr int kHostSteps = 16;                         // groups when the caller leaves the choice to the library
constexpr size_t kHostStagingBytes = size_t(1) << 30;  // staging cap for the library's choice

}  // namespace

extern "C" int sol_attn_forward_host(const void* q, const void* k, const void* v, void* out, int dtype, int batch,
                                     int heads, int L, int d, int Bq, int Bk, float beta, unsigned int flags,
                                     int slices_per_step, void* stream) {
  if (dtype != SOL_DTYPE_BF16 && dtype != SOL_DTYPE_F32) return SOL_ERR_INVALID_ARG;
  if (flags & ~(SOL_FLAG_KEEP_OR_DROP | SOL_FLAG_DIAGONAL_SIGMA | SOL_FLAG_ROUTE_IN_KERNEL))
    return SOL_ERR_INVALID_ARG;
  if (slices_per_step < 0) return SOL_ERR_INVALID_ARG;
  Geometry g;
  int rc = check_args(q, k, v, out, batch, heads, L, d, Bq, Bk, beta, &g);
  if (rc != SOL_OK) return rc;
  if ((flags & SOL_FLAG_ROUTE_IN_KERNEL) && !inkernel_supported(dtype, g)) return SOL_ERR_UNSUPPORTED;
  const size_t slice = (size_t)L * d * (dtype == SOL_DTYPE_BF16 ? 2 : 4);  // bytes of one (batch, head) slice
  int G = slices_per_step;
  if (G == 0) {
    G = (g.bH + kHostSteps - 1) / kHostSteps;
    const size_t cap = kHostStagingBytes / (8 * slice);  // two buffers of q, k, v, out
    if ((size_t)G > cap) G = cap > 0 ? (int)cap : 1;
  }
  if (G > g.bH) G = g.bH;
  const int steps = (g.bH + G - 1) / G;
  const size_t group = slice * G;  // bytes of one tensor's group
  HostStreams hs;
  if ((rc = host_streams(&hs)) != SOL_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  cudaEvent_t ev[9] = {};  // start, in[2], comp[2], out[2], end[2]
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      for (auto& x : ev)
        if (x) cudaEventDestroy(x);
      cudaGetLastError();
      return SOL_ERR_CUDA;
    }
  cudaEvent_t ev_start = ev[0], *ev_in = ev + 1, *ev_comp = ev + 3, *ev_out = ev + 5, *ev_end = ev + 7;
  void* staging = nullptr;
  if (scratch_alloc(&staging, 2 * 4 * group, st) != cudaSuccess) {
    for (auto& x : ev) cudaEventDestroy(x);
    cudaGetLastError();
    return SOL_ERR_NO_MEMORY;
  }
  // staging buffer b: q, k, v, out groups back to back
  auto buf = [&](int b, int t) { return static_cast<char*>(staging) + (size_t)(4 * b + t) * group; };
  const char* hin[3] = {static_cast<const char*>(q), static_cast<const char*>(k), static_cast<const char*>(v)};
  cudaError_t e = cudaEventRecord(ev_start, st);  // after the staging allocation and the caller's earlier work
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.h2d, ev_start, 0);
  for (int c = 0; c < steps && e == cudaSuccess && rc == SOL_OK; ++c) {
    const int b = c & 1;
    const int n = c == steps - 1 ? g.bH - c * G : G;  // slices in this group
    const size_t off = slice * (size_t)c * G, bytes = slice * n;
    // inputs of group c, once group c - 2 no longer reads buffer b
    if (c >= 2) e = cudaStreamWaitEvent(hs.h2d, ev_comp[b], 0);
    for (int t = 0; t < 3 && e == cudaSuccess; ++t)
      e = cudaMemcpyAsync(buf(b, t), hin[t] + off, bytes, cudaMemcpyHostToDevice, hs.h2d);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[b], hs.h2d);
    // compute, once the inputs are in and group c - 2's output has left buffer b
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_in[b], 0);
    if (e == cudaSuccess && c >= 2) e = cudaStreamWaitEvent(st, ev_out[b], 0);
    if (e != cudaSuccess) break;
    rc = forward_impl(buf(b, 0), buf(b, 1), buf(b, 2), buf(b, 3), dtype, 1, n, L, d, Bq, Bk, beta, flags, nullptr,
                      st);
    if (rc != SOL_OK) break;
    e = cudaEventRecord(ev_comp[b], st);
    // output of group c
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.d2h, ev_comp[b], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(out) + off, buf(b, 3), bytes, cudaMemcpyDeviceToHost, hs.d2h);
    if (e == cudaSuccess) e = cudaEventRecord(ev_out[b], hs.d2h);
  }
  // the caller's stream goes on only after everything enqueued on the
  // internal streams (every copy back, and any copy in left by an error):
  // the staging memory is freed after them
  for (int t = 0; t < 2; ++t) {
    cudaStream_t is = t ? hs.d2h : hs.h2d;
    cudaError_t e2 = cudaEventRecord(ev_end[t], is);
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, ev_end[t], 0);
    if (e == cudaSuccess) e = e2;
  }
  cudaFreeAsync(staging, st);
  for (auto& x : ev) cudaEventDestroy(x);  // released once their pending records complete
  if (rc != SOL_OK) return rc;
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SOL_ERR_CUDA;
  }
  return SOL_OK;
}
