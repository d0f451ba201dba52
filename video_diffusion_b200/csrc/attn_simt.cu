// attn_simt.cu -- the Sol-Attn attention loop on CUDA cores, fp32 arithmetic.
//
// Runs float32 inputs (where the tolerance asks for fp32 accuracy that bf16
// tensor-core operands cannot give) and the shapes the tensor-core kernel is
// not built for.  Same Eq. 9/10 folding as the tensor-core kernel: the pooled
// keys of unselected blocks first (logit q.K-bar_j / sqrt(d) + ln n_j, value
// V-hat_j / n_j), then every selected key block in increasing order, all
// merged into one exact per-row online softmax (running max, denominator,
// accumulator).
//
// One CTA per work item (query block), one thread per query row; key tiles
// pass through shared memory KT rows at a time.
#include <cmath>
#include <cstdint>

#include "common.cuh"

namespace sol {
namespace {

constexpr int KT = 32;  // key rows staged per sub-tile

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

template <typename T, int D, int BQ>
constexpr size_t simt_smem_bytes() { return sizeof(float) * ((size_t)(BQ + KT) * (D + 1) + KT * D); }

// One CTA of BQ threads per work item (query block); thread r owns query row r.
// Key blocks hold Bk tokens (the last nk_last); pooled keys pass through
// shared memory KT at a time, key blocks KT rows at a time.
template <typename T, int D, int BQ>
__global__ void __launch_bounds__(BQ) attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       const T* __restrict__ v, const float* __restrict__ kbar,
                                                       const float* __restrict__ vbar,
                                                       const uint32_t* __restrict__ mask,
                                                       const int32_t* __restrict__ order, int L, int Nq, int Bk,
                                                       int Nk, int W, int correction, float scale,
                                                       T* __restrict__ out) {
  extern __shared__ float sm[];
  float (*qs)[D + 1] = reinterpret_cast<float (*)[D + 1]>(sm);
  float (*ks)[D + 1] = reinterpret_cast<float (*)[D + 1]>(sm + BQ * (D + 1));
  float (*vs)[D] = reinterpret_cast<float (*)[D]>(sm + (BQ + KT) * (D + 1));
  const int item = order[blockIdx.x];
  const int bh = item / Nq, qi = item % Nq;
  const int r = threadIdx.x;
  const int n_rows = min(BQ, L - qi * BQ);
  const int nk_last = L - (Nk - 1) * Bk;
  const size_t head = (size_t)bh * L * D;
  const uint32_t* mrow = mask + (size_t)item * W;
  const float ln_full = logf((float)Bk), ln_last = logf((float)nk_last);
  auto selected = [&](int j) { return ((mrow[j >> 5] >> (j & 31)) & 1u) != 0u; };

  for (int e = r; e < BQ * D; e += BQ) {
    const int rr = e / D, c = e % D;
    qs[rr][c] = rr < n_rows ? ld_f(q + head + (size_t)(qi * BQ + rr) * D + c) : 0.f;
  }

  float acc[D];
#pragma unroll
  for (int c = 0; c < D; ++c) acc[c] = 0.f;
  float m = -INFINITY, l = 0.f;

  // columns [0, ncols) of the staged sub-tile; column c is pooled key base + c
  // when approx, else a token of the current key block
  auto fold_tile = [&](int ncols, bool approx, int base) {
    for (int c = 0; c < ncols; ++c) {
      float bias = 0.f;
      if (approx) {
        const int j = base + c;
        if (selected(j)) continue;  // selected: attended exactly
        bias = (j == Nk - 1) ? ln_last : ln_full;
      }
      float x = 0.f;
#pragma unroll 16
      for (int dd = 0; dd < D; ++dd) x = fmaf(qs[r][dd], ks[c][dd], x);
      x = fmaf(x, scale, bias);
      if (x > m) {
        const float corr = expf(m - x);
        l *= corr;
#pragma unroll
        for (int dd = 0; dd < D; ++dd) acc[dd] *= corr;
        m = x;
      }
      const float w = expf(x - m);
      l += w;
#pragma unroll
      for (int dd = 0; dd < D; ++dd) acc[dd] = fmaf(w, vs[c][dd], acc[dd]);
    }
  };

  // pooled keys of the unselected blocks (Eqs. 9-10), KT at a time
  if (correction) {
    for (int s0 = 0; s0 < Nk; s0 += KT) {
      const int nc = min(KT, Nk - s0);
      bool any = false;
      for (int c = 0; c < nc; ++c) any |= !selected(s0 + c);
      if (!any) continue;
      __syncthreads();
      const float* kb = kbar + ((size_t)bh * Nk + s0) * D;
      const float* vb = vbar + ((size_t)bh * Nk + s0) * D;
      for (int e = r; e < nc * D; e += BQ) {
        ks[e / D][e % D] = kb[e];
        vs[e / D][e % D] = vb[e];
      }
      __syncthreads();
      fold_tile(nc, true, s0);
    }
  }
  // selected blocks
  for (int w = 0; w < W; ++w) {
    uint32_t bits = mrow[w];
    while (bits) {
      const int j = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
      const int nj = min(Bk, L - j * Bk);
      for (int s0 = 0; s0 < nj; s0 += KT) {
        const int nc = min(KT, nj - s0);
        __syncthreads();
        const T* kp = k + head + ((size_t)j * Bk + s0) * D;
        const T* vp = v + head + ((size_t)j * Bk + s0) * D;
        for (int e = r; e < nc * D; e += BQ) {
          ks[e / D][e % D] = ld_f(kp + e);
          vs[e / D][e % D] = ld_f(vp + e);
        }
        __syncthreads();
        fold_tile(nc, false, 0);
      }
    }
  }
  if (r < n_rows) {
    const float inv = l > 0.f ? 1.0f / l : 0.f;  // nothing attended (keep-or-drop, no block selected): 0
    T* o = out + head + (size_t)(qi * BQ + r) * D;
#pragma unroll
    for (int dd = 0; dd < D; ++dd) st_f(o + dd, acc[dd] * inv);
  }
}

template <typename T>
cudaError_t dispatch(const void* q, const void* k, const void* v, void* out, const Geometry& g, const Scratch& s,
                     cudaStream_t st, int correction) {
  const float scale = 1.0f / sqrtf((float)g.d);
#define SOL_SIMT_CASE(D_, BQ_)                                                                                 \
  if (g.d == D_ && g.Bq == BQ_) {                                                                              \
    const size_t smem = simt_smem_bytes<T, D_, BQ_>();                                                         \
    cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D_, BQ_>,                                         \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);             \
    if (e != cudaSuccess) return e;                                                                            \
    attn_simt_kernel<T, D_, BQ_><<<g.nitems, BQ_, smem, st>>>(                                                 \
        (const T*)q, (const T*)k, (const T*)v, s.kbar, (const float*)s.vbar_op, s.mask, s.order, g.L, g.Nq,     \
        g.Bk, g.Nk, g.W, correction, scale, (T*)out);                                                          \
    return cudaGetLastError();                                                                                 \
  }
  SOL_SIMT_CASE(64, 64)
  SOL_SIMT_CASE(64, 128)
  SOL_SIMT_CASE(128, 64)
  SOL_SIMT_CASE(128, 128)
#undef SOL_SIMT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

// dtype: 0 = bf16, 1 = fp32.  K-bar (fp32) and V-bar (fp32) come from the pool kernel.
cudaError_t launch_attn_simt(int dtype, const void* q, const void* k, const void* v, void* out,
                             const Geometry& g, const Scratch& s, cudaStream_t st, int correction) {
  if (dtype == 1) return dispatch<float>(q, k, v, out, g, s, st, correction);
  return dispatch<__nv_bfloat16>(q, k, v, out, g, s, st, correction);
}

}  // namespace sol
