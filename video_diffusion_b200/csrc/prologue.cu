// prologue.cu -- block pooling, proxy scores, Eq. 4 routing and the work order.
//
// Sol-Attn visual explainer (mxino.github.io):
//   "Pool Q, K and V into blocks" -> pool_kernel: Q-bar_i, K-bar_j are block
//     means, V-hat_j the block sum (stored divided by n_j, with log n_j added to
//     the pooled logit by the attention kernel: n_j e^a V-hat_j/n_j / (n_j e^a)).
//   Eq. 4 / Eq. 5 -> route_blk_kernel (route_kernel for very long rows): the
//     proxy row s_i = Q-bar_i K-bar^T / sqrt(d) is formed on chip (shared
//     memory), and route_rows takes its mean and population standard
//     deviation to tau_i = mu_i + beta sigma_i; S_i = {j : s_ij > tau_i}
//     leaves as one bit per pair.  No Nq x Nk score map reaches global memory.
//     The diagonal estimator named beside Eq. 5 (kvar_kernel + route_rows)
//     takes sigma_i from the per-channel variances of K-bar instead.
// All reductions run in a fixed order, so results are deterministic.
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace sol {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr int kPoolThreads = 256;

// Sum of the rows [r0, r0 + n) of X ([rows, D] slice of one head), one 16-byte
// column group per thread: thread (cg, rl) adds rows rl, rl + R, ... of its
// group; the R partial sums are then added in shared memory in fixed order.
template <typename T, int D>
__device__ void block_column_sums(const T* __restrict__ X, int n, float* __restrict__ red, float* __restrict__ out) {
  constexpr int VEC = 16 / sizeof(T);   // elements per 16-byte load
  constexpr int G = D / VEC;            // column groups per row
  constexpr int R = kPoolThreads / G;   // row lanes
  const int tid = threadIdx.x;
  const int cg = tid % G, rl = tid / G;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  // Issue several independent 16-byte loads before adding them.
  constexpr int U = 4;
  int r = rl;
  for (; r + (U - 1) * R < n; r += U * R) {
    uint4 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      raw[u] = __ldcs(reinterpret_cast<const uint4*>(X + (size_t)(r + u * R) * D) + cg);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const T* e8 = reinterpret_cast<const T*>(&raw[u]);
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] += to_f(e8[e]);
    }
  }
  for (; r < n; r += R) {
    uint4 raw = __ldcs(reinterpret_cast<const uint4*>(X + (size_t)r * D) + cg);
    const T* e8 = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += to_f(e8[e]);
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[rl * D + cg * VEC + e] = acc[e];
  __syncthreads();
  for (int c = tid; c < D; c += kPoolThreads) {
    float s = 0.f;
    for (int q = 0; q < R; ++q) s += red[q * D + c];
    out[c] = s;
  }
  __syncthreads();
}

// grid (max(Nq, Nk), bH).  CTA x pools query block x (Q-bar, fp32) if x < Nq
// and key block x (K-bar in fp32 and in the operand type, V-hat/n in the
// operand type) if x < Nk.
template <typename T, typename Op, int D>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                            const T* __restrict__ v, int L, int Bq, int Nq,
                                                            int Bk, int Nk, float* __restrict__ qbar,
                                                            float* __restrict__ kbar, Op* __restrict__ kbar_op,
                                                            Op* __restrict__ vbar_op) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int R = kPoolThreads / (D / VEC);
  __shared__ float red[R * D];
  __shared__ float sums[D];
  const int blk = blockIdx.x, bh = blockIdx.y;
  const size_t head = (size_t)bh * L * D;

  if (blk < Nq) {
    const int r0 = blk * Bq;
    const float inv_n = 1.0f / (float)min(Bq, L - r0);
    block_column_sums<T, D>(q + head + (size_t)r0 * D, min(Bq, L - r0), red, sums);
    const size_t prow = ((size_t)bh * Nq + blk) * D;
    for (int c = threadIdx.x; c < D; c += kPoolThreads) qbar[prow + c] = sums[c] * inv_n;
  }
  if (blk < Nk) {
    const int r0 = blk * Bk;
    const int n = min(Bk, L - r0);
    const float inv_n = 1.0f / (float)n;
    const size_t prow = ((size_t)bh * Nk + blk) * D;
    block_column_sums<T, D>(k + head + (size_t)r0 * D, n, red, sums);
    for (int c = threadIdx.x; c < D; c += kPoolThreads) {
      float m = sums[c] * inv_n;
      kbar[prow + c] = m;
      if (kbar_op) kbar_op[prow + c] = from_f<Op>(m);
    }
    if (v != nullptr) {
      block_column_sums<T, D>(v + head + (size_t)r0 * D, n, red, sums);
      for (int c = threadIdx.x; c < D; c += kPoolThreads) vbar_op[prow + c] = from_f<Op>(sums[c] * inv_n);
    }
  }
}

// grid (bH), 256 threads.  kvar[bh, c] = population variance over the Nk key
// blocks of K-bar_{j,c}, two passes (mean, then mean squared deviation); the
// per-thread partial sums are added in a fixed order.
template <int D>
__global__ void __launch_bounds__(256) kvar_kernel(const float* __restrict__ kbar, int Nk,
                                                   float* __restrict__ kvar) {
  constexpr int R = 256 / D;
  __shared__ float red[256];
  __shared__ float mean_s[D];
  const int bh = blockIdx.x, c = threadIdx.x % D, rl = threadIdx.x / D;
  const float* kb = kbar + (size_t)bh * Nk * D;
  float a = 0.f;
  for (int j = rl; j < Nk; j += R) a += kb[(size_t)j * D + c];
  red[threadIdx.x] = a;
  __syncthreads();
  if (threadIdx.x < D) {
    float t = 0.f;
    for (int r = 0; r < R; ++r) t += red[r * D + c];
    mean_s[c] = t / (float)Nk;
  }
  __syncthreads();
  const float m = mean_s[c];
  float v = 0.f;
  for (int j = rl; j < Nk; j += R) {
    const float t = kb[(size_t)j * D + c] - m;
    v = fmaf(t, t, v);
  }
  red[threadIdx.x] = v;
  __syncthreads();
  if (threadIdx.x < D) {
    float t = 0.f;
    for (int r = 0; r < R; ++r) t += red[r * D + c];
    kvar[(size_t)bh * D + c] = t / (float)Nk;
  }
}

constexpr int kRouteThreads = 256;
constexpr int kRouteKC = 32;  // pooled keys staged in shared memory at a time
template <int D>
constexpr int route_ks_stride() { return D + 4; }  // 16-byte rows, and rows 4 banks apart

// Row pass of the router for the score rows srow[qi * NS + j] (qi < nq,
// j < Nk) of query blocks i0 .. i0 + nq - 1 of head bh: warp w of the
// NTHREADS / 32 takes rows w, w + NTHREADS / 32, ...  qrows[qi * qstride ..] is Q-bar of row qi (diagonal estimator only).
// kvar == nullptr: sigma_i from the row (Eq. 5); else the diagonal estimator.
// tiles[i] counts the attention kernel's tiles: pooled-key chunks used plus the
// selected blocks, two to a tile when pair != 0.  mask and tau_out may be null.
template <int D, int NTHREADS>
__device__ void route_rows(const float* srow, int NS, const float* qrows, int qstride, int bh, int i0, int nq,
                           int Nq, int Nk,
                           int W, float scale, float beta, int beta_mode, int correction, int pair,
                           const float* __restrict__ kvar, uint32_t* __restrict__ mask,
                           int32_t* __restrict__ counts, int32_t* __restrict__ tiles, float* __restrict__ tau_out,
                           int32_t* __restrict__ near, float near_margin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int qi = warp; qi < nq; qi += NTHREADS / 32) {
    const float* s = srow + (size_t)qi * NS;
    // mean and population variance, two passes, lane-strided then a fixed tree
    float a = 0.f;
    for (int j = lane; j < Nk; j += 32) a += s[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    const float mu = a / (float)Nk;
    float v = 0.f;
    if (kvar == nullptr) {
      for (int j = lane; j < Nk; j += 32) {
        float t = s[j] - mu;
        v = fmaf(t, t, v);
      }
    } else {
      const float* qv = qrows + (size_t)qi * qstride;
      const float* kvh = kvar + (size_t)bh * D;
      for (int c = lane; c < D; c += 32) v = fmaf(qv[c] * qv[c], kvh[c], v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const float sigma = kvar == nullptr ? sqrtf(v / (float)Nk) : scale * sqrtf(v);
    float tau;
    if (beta_mode < 0) tau = -INFINITY;
    else if (beta_mode > 0) tau = INFINITY;
    else tau = fmaf(beta, sigma, mu);

    const size_t item = (size_t)bh * Nq + i0 + qi;
    // one mask word per step: lane l tests key block 32w + l (consecutive
    // shared-memory reads), a ballot gathers the word; a pooled-key chunk
    // (kChunk / 32 words) counts as a tile if it holds an unselected block
    constexpr int wpc = kChunk / 32;
    int cnt = 0, used = 0;
    bool chunk_has_unselected = false;
    for (int w = 0; w < W; ++w) {
      const int j = w * 32 + lane;
      const bool valid = j < Nk;
      const uint32_t word = __ballot_sync(0xffffffffu, valid && s[j] > tau);
      const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
      if (mask && lane == 0) mask[item * W + w] = word;
      cnt += __popc(word);
      chunk_has_unselected |= ((~word) & vmask) != 0u;
      if (w % wpc == wpc - 1 || w == W - 1) {
        used += chunk_has_unselected ? 1 : 0;
        chunk_has_unselected = false;
      }
    }
    if (!correction) used = 0;
    if (lane == 0) {
      counts[item] = cnt;
      tiles[item] = (pair ? (cnt + 1) >> 1 : cnt) + used;
      if (tau_out) tau_out[item] = tau;
    }
    if (near) {  // diagnostics only: decisions within near_margin of tau_i
      int nt = 0;
      for (int j = lane; j < Nk; j += 32) nt += fabsf(s[j] - tau) < near_margin ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nt += __shfl_xor_sync(0xffffffffu, nt, o);
      if (lane == 0) near[item] = nt;
    }
  }
}

// Router for any Nk the shared memory holds at QB = 8 * QPW rows (up to 32).
// grid (ceil(Nq / QB), bH), 256 threads.  Score pass: lane l takes staged key
// l, warp w the query blocks w*QB/8 .. (w+1)*QB/8 - 1, so each thread runs
// QB/8 independent dot products over one key row.
template <int D, int QPW>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              const float* __restrict__ kvar, int Nq, int Nk,
                                                              int W, float scale, float beta, int beta_mode,
                                                              int correction, int pair, uint32_t* __restrict__ mask,
                                                              int32_t* __restrict__ counts,
                                                              int32_t* __restrict__ tiles,
                                                              float* __restrict__ tau_out,
                                                              int32_t* __restrict__ near, float near_margin) {
  constexpr int QB = 8 * QPW;
  extern __shared__ float sm[];
  float* qs = sm;                          // [QB][D]
  constexpr int KS = route_ks_stride<D>();
  float* ks = qs + QB * D;                 // [KC][KS]
  float* srow = ks + kRouteKC * KS;        // [QB][Nk]
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * QB;
  const int nq = min(QB, Nq - i0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* qb = qbar + ((size_t)bh * Nq + i0) * D;
  const float* kb = kbar + (size_t)bh * Nk * D;

  for (int e = tid; e < QB * D; e += kRouteThreads) qs[e] = e < nq * D ? qb[e] : 0.f;
  for (int j0 = 0; j0 < Nk; j0 += kRouteKC) {
    const int nk = min(kRouteKC, Nk - j0);
    __syncthreads();
    for (int e = tid; e < nk * D; e += kRouteThreads) {
      int jj = e / D, c = e % D;
      ks[jj * KS + c] = kb[(size_t)(j0 + jj) * D + c];
    }
    __syncthreads();
    if (lane < nk) {
      const float* kv = ks + lane * KS;
      const float* qv = qs + warp * QPW * D;
      float acc[QPW];
#pragma unroll
      for (int q = 0; q < QPW; ++q) acc[q] = 0.f;
      // four channels per 16-byte load (the query rows are broadcast to the
      // warp); each sum still takes its channels in order, one fused
      // multiply-add each, as the attention kernel's in-kernel routing does
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        const float4 k4 = *reinterpret_cast<const float4*>(kv + c);
#pragma unroll
        for (int q = 0; q < QPW; ++q) {
          const float4 q4 = *reinterpret_cast<const float4*>(qv + q * D + c);
          acc[q] = fmaf(q4.x, k4.x, acc[q]);
          acc[q] = fmaf(q4.y, k4.y, acc[q]);
          acc[q] = fmaf(q4.z, k4.z, acc[q]);
          acc[q] = fmaf(q4.w, k4.w, acc[q]);
        }
      }
#pragma unroll
      for (int q = 0; q < QPW; ++q) {
        const int qi = warp * QPW + q;
        if (qi < nq) srow[(size_t)qi * Nk + j0 + lane] = acc[q] * scale;
      }
    }
  }
  __syncthreads();
  route_rows<D, kRouteThreads>(srow, Nk, qs, D, bh, i0, nq, Nq, Nk, W, scale, beta, beta_mode, correction, pair, kvar, mask,
                counts, tiles, tau_out, near, near_margin);
}

__device__ __forceinline__ void cp_async16(float* smem_dst, const float* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kBlkKC = 128;  // register-blocked router: pooled keys staged per chunk (32 per warp)

// Score-row stride of the register-blocked router: at least Nk and 8 banks
// past a multiple of 32, so that the four rows a warp stores to at once fall
// in different banks.
__host__ __device__ inline int blk_row_stride(int Nk) { return Nk + ((8 - Nk) & 31); }

// Router for Nk up to what QH * 16 score rows leave room for (QH = 2: about
// 1100 pooled keys at d = 128; QH = 1: about 2400).  grid (ceil(Nq / (16 QH)),
// bH), 128 QH threads: QH groups of four warps, group h taking query blocks
// 16h .. 16h + 15 of the CTA's.  Score pass: register-blocked like a small
// matrix product; lane (tq, tk) = (lane / 8, lane % 8) of warp w of a group
// computes its query blocks tq + 4a (a < 4) against keys 32w + tk + 8b (b < 4)
// of each staged chunk of 128 (the chunk serves all QH groups), so per four
// channels it
// makes 8 16-byte shared-memory loads (4 of query rows, 4 of key rows, each
// shared by a group of lanes, conflict-free) for 64 fused multiply-adds.  Each
// score is the same sequence of fused multiply-adds over the channels in
// order, then the 1/sqrt(d) scale, as in route_kernel and the attention
// kernel's in-kernel routing, so all three give the same bits.
template <int D, int QH>
__global__ void __launch_bounds__(128 * QH) route_blk_kernel(
    const float* __restrict__ qbar, const float* __restrict__ kbar, const float* __restrict__ kvar, int Nq, int Nk,
    int NS, int W, float scale, float beta, int beta_mode, int correction, int pair, uint32_t* __restrict__ mask,
    int32_t* __restrict__ counts, int32_t* __restrict__ tiles, float* __restrict__ tau_out,
    int32_t* __restrict__ near, float near_margin) {
  constexpr int RS = route_ks_stride<D>();  // shared-memory row stride of Q-bar and K-bar rows
  constexpr int QB = 16 * QH, NT = 128 * QH;
  extern __shared__ __align__(16) float blk_sm[];
  float* qs = blk_sm;                 // [QB][RS]
  float* ks = qs + QB * RS;           // [128][RS]
  float* srow = ks + kBlkKC * RS;     // [QB][NS]
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * QB;
  const int nq = min(QB, Nq - i0);
  const int tid = threadIdx.x, lane = tid & 31;
  const int qg = tid >> 7, warp = (tid >> 5) & 3;  // query group, warp within the group
  const int tq = lane >> 3, tk = lane & 7;
  const float* qb = qbar + ((size_t)bh * Nq + i0) * D;
  const float* kb = kbar + (size_t)bh * Nk * D;

  // rows past nq repeat the last row; their scores are not stored
  for (int e = tid; e < QB * (D / 4); e += NT) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    cp_async16(qs + r * RS + 4 * c4, qb + (size_t)min(r, nq - 1) * D + 4 * c4);
  }
  for (int j0 = 0; j0 < Nk; j0 += kBlkKC) {
    const int nk = min(kBlkKC, Nk - j0);
    __syncthreads();  // the previous chunk has been read by every warp
    for (int e = tid; e < nk * (D / 4); e += NT) {
      const int r = e / (D / 4), c4 = e % (D / 4);
      cp_async16(ks + r * RS + 4 * c4, kb + (size_t)(j0 + r) * D + 4 * c4);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    const int kw = warp * 32;  // this warp's 32 keys of the chunk
    if (kw < nk) {
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
      const float* qr = qs + (16 * qg + tq) * RS;
      const float* kr = ks + (kw + tk) * RS;  // key rows past nk hold stale data, never stored
#pragma unroll 2
      for (int c = 0; c < D; c += 4) {
        float4 q4[4], k4[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) q4[a] = *reinterpret_cast<const float4*>(qr + 4 * a * RS + c);
#pragma unroll
        for (int b = 0; b < 4; ++b) k4[b] = *reinterpret_cast<const float4*>(kr + 8 * b * RS + c);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            acc[a][b] = fmaf(q4[a].x, k4[b].x, acc[a][b]);
            acc[a][b] = fmaf(q4[a].y, k4[b].y, acc[a][b]);
            acc[a][b] = fmaf(q4[a].z, k4[b].z, acc[a][b]);
            acc[a][b] = fmaf(q4[a].w, k4[b].w, acc[a][b]);
          }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const int qi = 16 * qg + tq + 4 * a;
        if (qi < nq) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int jj = kw + tk + 8 * b;
            if (jj < nk) srow[(size_t)qi * NS + j0 + jj] = acc[a][b] * scale;
          }
        }
      }
    }
  }
  __syncthreads();
  route_rows<D, NT>(srow, NS, qs, RS, bh, i0, nq, Nq, Nk, W, scale, beta, beta_mode, correction, pair, kvar, mask,
                    counts, tiles, tau_out, near, near_margin);
}

// One CTA per head: bitonic sort of the head's work items by (tiles desc,
// index asc); writes order[bh * NI + rank] = bh * NI + i.  A work item is G
// consecutive query blocks (G = 1, or 2 for 64-token blocks that share a
// 128-row tile; NI = ceil(N / G) items per head), weighed by the sum of its
// blocks' tile counts.
__global__ void __launch_bounds__(1024) order_kernel(const int32_t* __restrict__ tiles, int N, int G, int P,
                                                     int32_t* __restrict__ order) {
  extern __shared__ unsigned long long keys[];
  const int bh = blockIdx.x;
  const int NI = (N + G - 1) / G;
  for (int e = threadIdx.x; e < P; e += blockDim.x) {
    unsigned long long key;
    if (e < NI) {
      uint32_t t = 0;
      for (int q = G * e; q < G * e + G && q < N; ++q) t += (uint32_t)tiles[(size_t)bh * N + q];
      key = ((unsigned long long)(0x7fffffffu - t) << 32) | (uint32_t)e;
    } else {
      key = ~0ull;
    }
    keys[e] = key;
  }
  __syncthreads();
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int e = threadIdx.x; e < P; e += blockDim.x) {
        const int partner = e ^ stride;
        if (partner > e) {
          const bool up = (e & size) == 0;
          unsigned long long a = keys[e], b = keys[partner];
          if ((a > b) == up) {
            keys[e] = b;
            keys[partner] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < NI; e += blockDim.x)
    order[(size_t)bh * NI + e] = bh * NI + (int)(uint32_t)(keys[e] & 0xffffffffu);
}

__global__ void identity_order_kernel(int32_t* order, int n) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) order[e] = e;
}

template <typename T, typename Op>
cudaError_t pool_dispatch(const void* q, const void* k, const void* v, const Geometry& g, const Scratch& s,
                          cudaStream_t st) {
  dim3 grid(g.Nq > g.Nk ? g.Nq : g.Nk, g.bH);
  if (g.d == 128)
    pool_kernel<T, Op, 128><<<grid, kPoolThreads, 0, st>>>((const T*)q, (const T*)k, (const T*)v, g.L, g.Bq,
                                                           g.Nq, g.Bk, g.Nk, s.qbar, s.kbar, (Op*)s.kbar_op,
                                                           (Op*)s.vbar_op);
  else
    pool_kernel<T, Op, 64><<<grid, kPoolThreads, 0, st>>>((const T*)q, (const T*)k, (const T*)v, g.L, g.Bq,
                                                          g.Nq, g.Bk, g.Nk, s.qbar, s.kbar, (Op*)s.kbar_op,
                                                          (Op*)s.vbar_op);
  return cudaGetLastError();
}

}  // namespace

// in_dtype / op_dtype: 0 = bf16, 1 = fp32.
cudaError_t launch_pool(int in_dtype, int op_dtype, const void* q, const void* k, const void* v,
                        const Geometry& g, const Scratch& s, cudaStream_t st) {
  if (in_dtype == 0 && op_dtype == 0) return pool_dispatch<__nv_bfloat16, __nv_bfloat16>(q, k, v, g, s, st);
  if (in_dtype == 0 && op_dtype == 1) return pool_dispatch<__nv_bfloat16, float>(q, k, v, g, s, st);
  if (in_dtype == 1 && op_dtype == 1) return pool_dispatch<float, float>(q, k, v, g, s, st);
  return pool_dispatch<float, __nv_bfloat16>(q, k, v, g, s, st);
}

// Query blocks per CTA (QB = 8 * QPW), bounded by the shared memory their
// score rows take.
static int route_qpw(int Nk) {
  int qpw = 4;
  while (qpw > 1 && (size_t)8 * qpw * Nk * sizeof(float) > 160u * 1024u) qpw >>= 1;
  return qpw;
}

template <int D, int QPW>
static cudaError_t route_launch(const Geometry& g, const Scratch& s, float beta, int beta_mode, int correction,
                                int pair, const float* kvar, cudaStream_t st) {
  constexpr int QB = 8 * QPW;
  const size_t smem = (size_t)(QB * D + kRouteKC * route_ks_stride<D>() + (size_t)QB * g.Nk) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(route_kernel<D, QPW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((g.Nq + QB - 1) / QB, g.bH);
  route_kernel<D, QPW><<<grid, kRouteThreads, smem, st>>>(s.qbar, s.kbar, kvar, g.Nq, g.Nk, g.W,
                                                          1.0f / sqrtf((float)D), beta, beta_mode, correction,
                                                          pair, s.mask, s.counts, s.tiles, s.tau, s.near,
                                                          s.near_margin);
  return cudaGetLastError();
}

constexpr size_t kRouteSmemMax = 227 * 1024;

template <int D>
static size_t route_blk_smem(int Nk, int qh) {
  return (size_t)((16 * qh + kBlkKC) * route_ks_stride<D>() + (size_t)16 * qh * blk_row_stride(Nk)) * sizeof(float);
}

template <int D, int QH>
static cudaError_t route_blk_launch(const Geometry& g, const Scratch& s, float beta, int beta_mode, int correction,
                                    int pair, const float* kvar, cudaStream_t st) {
  const size_t smem = route_blk_smem<D>(g.Nk, QH);
  cudaError_t e = cudaFuncSetAttribute(route_blk_kernel<D, QH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((g.Nq + 16 * QH - 1) / (16 * QH), g.bH);
  route_blk_kernel<D, QH><<<grid, 128 * QH, smem, st>>>(s.qbar, s.kbar, kvar, g.Nq, g.Nk, blk_row_stride(g.Nk),
                                                        g.W, 1.0f / sqrtf((float)D), beta, beta_mode, correction,
                                                        pair, s.mask, s.counts, s.tiles, s.tau, s.near,
                                                        s.near_margin);
  return cudaGetLastError();
}

template <int D>
static cudaError_t route_dispatch(const Geometry& g, const Scratch& s, float beta, int beta_mode, int correction,
                                 int pair, const float* kvar, cudaStream_t st) {
  if (route_blk_smem<D>(g.Nk, 2) <= kRouteSmemMax)
    return route_blk_launch<D, 2>(g, s, beta, beta_mode, correction, pair, kvar, st);
  if (route_blk_smem<D>(g.Nk, 1) <= kRouteSmemMax)
    return route_blk_launch<D, 1>(g, s, beta, beta_mode, correction, pair, kvar, st);
  const int qpw = route_qpw(g.Nk);
  if (qpw == 4) return route_launch<D, 4>(g, s, beta, beta_mode, correction, pair, kvar, st);
  if (qpw == 2) return route_launch<D, 2>(g, s, beta, beta_mode, correction, pair, kvar, st);
  return route_launch<D, 1>(g, s, beta, beta_mode, correction, pair, kvar, st);
}

cudaError_t launch_route(const Geometry& g, const Scratch& s, float beta, int beta_mode, int correction,
                         int sigma_mode, int pair, cudaStream_t st) {
  const float* kvar = nullptr;
  if (sigma_mode == kSigmaDiagonal) {
    if (g.d == 128)
      kvar_kernel<128><<<g.bH, 256, 0, st>>>(s.kbar, g.Nk, s.kvar);
    else
      kvar_kernel<64><<<g.bH, 256, 0, st>>>(s.kbar, g.Nk, s.kvar);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    kvar = s.kvar;
  }
  if (g.d == 128) return route_dispatch<128>(g, s, beta, beta_mode, correction, pair, kvar, st);
  return route_dispatch<64>(g, s, beta, beta_mode, correction, pair, kvar, st);
}

cudaError_t launch_order(const Geometry& g, const Scratch& s, int group, cudaStream_t st) {
  const int NI = (g.Nq + group - 1) / group;
  if (NI > kOrderMaxN) {
    identity_order_kernel<<<148, 256, 0, st>>>(s.order, g.bH * NI);
    return cudaGetLastError();
  }
  int P = 1;
  while (P < NI) P <<= 1;
  const size_t smem = (size_t)P * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  order_kernel<<<g.bH, 1024, smem, st>>>(s.tiles, g.Nq, group, P, s.order);
  return cudaGetLastError();
}

}  // namespace sol
