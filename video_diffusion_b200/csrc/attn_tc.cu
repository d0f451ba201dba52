// attn_tc.cu -- the Sol-Attn attention loop on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), bf16 operands, fp32 accumulation, d = 128, B = 128.
//
// One online-softmax pass per query block i (Sol-Attn visual explainer, "One
// online-softmax state": exact and approximate terms share the running
// maximum, the denominator and the numerator):
//   * approximate tiles first -- for each chunk t of 128 pooled keys that holds
//     an unselected block, S~ = Q_i K-bar^(t)T (Eq. 11's token-to-block tile);
//     column j carries logit S~_j / sqrt(d) + ln n_j and value V-hat_j / n_j,
//     which is Eq. 9's n_j exp(.) and Eq. 10's exp(.) V-hat_j folded into one
//     softmax column; selected and out-of-range columns are masked out;
//   * then each selected key block j in increasing order: S = Q_i K_j^T, masked
//     past the block's n_j tokens, and O += P V_j (Eqs. 9, 10 "Exact" terms).
//     Only selected K/V tiles are ever loaded.
//
// Persistent CTAs, one per SM, 192 threads:
//   warp 0      TMA producer: Q tile, then K/V (or K-bar/V-bar) tiles in a
//               3-stage K ring and a 2-stage V ring; fetches work items
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//   warps 2..5  softmax: one query row per thread (TMEM lane), P to TMEM,
//               lazy O rescaling, epilogue
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
// Every mbarrier wait is bounded; on expiry the CTA abandons its work, waits
// for its own copies and MMAs, frees TMEM and records the failing wait in the
// device status word.
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace sol {

__device__ int g_sol_status;  // 0 = ok; else 0x1000 | wait id (first expiry)

namespace {

constexpr int BM = 128, BN = 128, HD = 128;
constexpr int KST = 3, VST = 2;
constexpr int NTHREADS = 192;
constexpr uint32_t TILE_BYTES = BM * HD * 2;  // 32 KB, two 64-column swizzled halves
constexpr uint32_t HALF_BYTES = TILE_BYTES / 2;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = TILE_BYTES;
constexpr uint32_t OFF_V = OFF_K + KST * TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_V + VST * TILE_BYTES;  // 192 KB
constexpr uint32_t SMEM_BYTES = OFF_BAR + 1024 + 1024;  // barriers + alignment slack

constexpr uint32_t TM_S = 0, TM_O = 256, TM_P = 384;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

struct Params {
  int bH, L, N, W, nchunk, nitems, n_last;
  float scale_log2;     // log2(e) / sqrt(d)
  float bias_full;      // log2(B)
  float bias_last;      // log2(n_last)
  const uint32_t* mask;
  const int32_t* tiles;
  const int32_t* order;
  int32_t* work_counter;
  __nv_bfloat16* out;
  uint64_t wait_limit_ns;
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];
  uint64_t pv_done[2];  // per P buffer: the PV MMA that read it has finished
  uint64_t o_full, o_free;
  uint64_t item_full[2], item_empty[2];
  uint64_t teardown;
  int item_slot[2];
  uint32_t tmem_base;
  int abort_flag;
};

// Walks the tile sequence of one work item: pooled-key chunks holding an
// unselected block, then the selected blocks in increasing order.
struct TileIter {
  const uint32_t* m;
  int W, N, nchunk;
  int chunk;     // next chunk to test
  int word;      // current mask word in the exact phase
  uint32_t bits; // remaining set bits of that word
  __device__ void init(const uint32_t* mrow, int W_, int N_, int nchunk_) {
    m = mrow; W = W_; N = N_; nchunk = nchunk_;
    chunk = 0; word = -1; bits = 0;
  }
  __device__ __forceinline__ uint32_t valid_bits(int w) const {
    const int nb = N - w * 32;
    return nb >= 32 ? 0xffffffffu : (nb <= 0 ? 0u : ((1u << nb) - 1u));
  }
  // kind 0: pooled chunk idx; kind 1: exact key block idx.  false when done.
  __device__ bool next(int& kind, int& idx) {
    while (chunk < nchunk) {
      const int c = chunk++;
      uint32_t un = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int w = c * 4 + q;
        if (w < W) un |= (~m[w]) & valid_bits(w);
      }
      if (un) { kind = 0; idx = c; return true; }
    }
    while (bits == 0) {
      if (++word >= W) return false;
      bits = m[word];
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1;
    kind = 1;
    idx = word * 32 + b;
    return true;
  }
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars& B_, uint64_t lim, int id) {
  return mbar_wait(bar, parity, &B_.abort_flag, &g_sol_status, 0x1000 | id, lim);
}
// All 32 lanes wait; the outcome is made warp-uniform so that the warp-wide
// tcgen05.ld/st that follow are never reached by part of a warp.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, Bars& B_, uint64_t lim, int id) {
  const bool ok = wait_bar(bar, parity, B_, lim, id);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------------------ softmax helpers
// u_c = s_c * scale_log2 + bias_c for valid columns, -inf otherwise; returns max.
template <bool FULL>
__device__ __forceinline__ float tile_logits(float (&x)[128], float sl2, float bias, const uint32_t (&vm)[4],
                                             int sc, float sc_delta) {
  float rmax = -INFINITY;
#pragma unroll
  for (int c = 0; c < 128; ++c) {
    float u = fmaf(x[c], sl2, bias);
    if (!FULL) {
      if (c == sc) u += sc_delta;
      if (!((vm[c >> 5] >> (c & 31)) & 1u)) u = -INFINITY;
    }
    x[c] = u;
    rmax = fmaxf(rmax, u);
  }
  return rmax;
}

__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                   const __grid_constant__ CUtensorMap tmVb, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < KST; ++s) { mbar_init(&bars.k_full[s], 1); mbar_init(&bars.k_empty[s], 1); }
    for (int s = 0; s < VST; ++s) { mbar_init(&bars.v_full[s], 1); mbar_init(&bars.v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_free[s], 4);
      mbar_init(&bars.p_full[s], 4);
      mbar_init(&bars.pv_done[s], 1);
      mbar_init(&bars.item_full[s], 1);
      mbar_init(&bars.item_empty[s], 5);
    }
    mbar_init(&bars.o_full, 1);
    mbar_init(&bars.o_free, 4);
    mbar_init(&bars.teardown, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmKb); tma_prefetch_desc(&tmVb);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t g = 0;          // global tile counter
      int it = 0;              // item counter
      int k_last_use[KST], v_last_use[VST], q_uses = 0;
      for (int s = 0; s < KST; ++s) k_last_use[s] = -1;
      for (int s = 0; s < VST; ++s) v_last_use[s] = -1;
      bool ok = true;
      for (;; ++it) {
        const int slot = it & 1;
        if (it >= 2 && !(ok = wait_bar(&bars.item_empty[slot], ((it >> 1) + 1) & 1, bars, lim, 1))) break;
        const int idx = atomicAdd(p.work_counter, 1);
        const int item = idx < p.nitems ? p.order[idx] : -1;
        bars.item_slot[slot] = item;
        mbar_arrive(&bars.item_full[slot]);
        if (item < 0) break;
        const int bh = item / p.N, qi = item % p.N;
        const int T = p.tiles[item];
        if (T == 0) continue;
        if (it > 0 && q_uses > 0 && !(ok = wait_bar(&bars.q_empty, (q_uses - 1) & 1, bars, lim, 2))) break;
        mbar_arrive_expect_tx(&bars.q_full, TILE_BYTES);
        tma_load_3d(smem + OFF_Q, &tmQ, &bars.q_full, 0, qi * BM, bh, pol_q);
        tma_load_3d(smem + OFF_Q + HALF_BYTES, &tmQ, &bars.q_full, 64, qi * BM, bh, pol_q);
        ++q_uses;
        TileIter ti;
        ti.init(p.mask + (size_t)item * p.W, p.W, p.N, p.nchunk);
        int pkind = 0, pidx = 0;
        for (int n = 0; n <= T && ok; ++n) {
          int kind = 0, tidx = 0;
          if (n < T) {
            ti.next(kind, tidx);
            const uint32_t gk = g + n;
            const int ks = gk % KST;
            if (gk >= KST && !(ok = wait_bar(&bars.k_empty[ks], ((gk / KST) + 1) & 1, bars, lim, 3))) break;
            uint8_t* dst = smem + OFF_K + ks * TILE_BYTES;
            mbar_arrive_expect_tx(&bars.k_full[ks], TILE_BYTES);
            const CUtensorMap* m = kind ? &tmK : &tmKb;
            tma_load_3d(dst, m, &bars.k_full[ks], 0, tidx * BN, bh, pol_kv);
            tma_load_3d(dst + HALF_BYTES, m, &bars.k_full[ks], 64, tidx * BN, bh, pol_kv);
            k_last_use[ks] = (int)(gk / KST);
          }
          if (n > 0) {
            const uint32_t gv = g + n - 1;
            const int vs = gv % VST;
            if (gv >= VST && !(ok = wait_bar(&bars.v_empty[vs], ((gv / VST) + 1) & 1, bars, lim, 4))) break;
            uint8_t* dst = smem + OFF_V + vs * TILE_BYTES;
            mbar_arrive_expect_tx(&bars.v_full[vs], TILE_BYTES);
            const CUtensorMap* m = pkind ? &tmV : &tmVb;
            tma_load_3d(dst, m, &bars.v_full[vs], 0, pidx * BN, bh, pol_kv);
            tma_load_3d(dst + HALF_BYTES, m, &bars.v_full[vs], 64, pidx * BN, bh, pol_kv);
            v_last_use[vs] = (int)(gv / VST);
          }
          pkind = kind;
          pidx = tidx;
        }
        if (!ok) break;
        g += T;
      }
      if (!ok || bars.abort_flag) {
        // let every copy this thread started land before the CTA exits
        for (int s = 0; s < KST; ++s)
          if (k_last_use[s] >= 0) mbar_wait(&bars.k_full[s], k_last_use[s] & 1, nullptr, &g_sol_status, 0, lim);
        for (int s = 0; s < VST; ++s)
          if (v_last_use[s] >= 0) mbar_wait(&bars.v_full[s], v_last_use[s] & 1, nullptr, &g_sol_status, 0, lim);
        if (q_uses > 0) mbar_wait(&bars.q_full, (q_uses - 1) & 1, nullptr, &g_sol_status, 0, lim);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
      const uint32_t sQ = smem_u32(smem + OFF_Q);
      const uint32_t sK = smem_u32(smem + OFF_K);
      const uint32_t sV = smem_u32(smem + OFF_V);
      uint32_t g = 0;
      int item_local = 0;  // items with T > 0 processed
      bool issued = false;
      bool ok = true;
      for (int it = 0;; ++it) {
        const int slot = it & 1;
        if (!(ok = wait_bar(&bars.item_full[slot], (it >> 1) & 1, bars, lim, 10))) break;
        const int item = bars.item_slot[slot];
        mbar_arrive(&bars.item_empty[slot]);
        if (item < 0) break;
        const int T = p.tiles[item];
        if (T == 0) continue;
        if (!(ok = wait_bar(&bars.q_full, item_local & 1, bars, lim, 11))) break;
        auto issue_pv = [&](uint32_t gp, bool first) -> bool {
          const int pb = gp & 1;
          if (!wait_bar(&bars.p_full[pb], (gp >> 1) & 1, bars, lim, 12)) return false;
          const int vs = gp % VST;
          if (!wait_bar(&bars.v_full[vs], (gp / VST) & 1, bars, lim, 13)) return false;
          if (first && item_local > 0 && !wait_bar(&bars.o_free, (item_local - 1) & 1, bars, lim, 14)) return false;
          tc_fence_after();
          const uint32_t vbase = sV + vs * TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(vbase + kk * 2048, HALF_BYTES, 1024);
            mma_ts(tmem + TM_O, tmem + TM_P + pb * 64 + kk * 8, bdesc, IDESC_PV, (first && kk == 0) ? 0u : 1u);
          }
          tc_commit(&bars.v_empty[vs]);
          tc_commit(&bars.pv_done[pb]);
          return true;
        };
        for (int n = 0; n < T && ok; ++n) {
          const uint32_t gs = g + n;
          const int ks = gs % KST;
          if (!(ok = wait_bar(&bars.k_full[ks], (gs / KST) & 1, bars, lim, 15))) break;
          const int sb = gs & 1;
          if (gs >= 2 && !(ok = wait_bar(&bars.s_free[sb], ((gs >> 1) + 1) & 1, bars, lim, 16))) break;
          tc_fence_after();
          const uint32_t kbase = sK + ks * TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
            const uint64_t adesc = smem_desc_sw128(sQ + off, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(kbase + off, 16, 1024);
            mma_ss(tmem + TM_S + sb * 128, adesc, bdesc, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          issued = true;
          tc_commit(&bars.s_full[sb]);
          tc_commit(&bars.k_empty[ks]);
          if (n == T - 1) tc_commit(&bars.q_empty);
          if (n > 0 && !(ok = issue_pv(gs - 1, n == 1))) break;
        }
        if (!ok) break;
        if (!(ok = issue_pv(g + T - 1, T == 1))) break;
        tc_commit(&bars.o_full);
        g += T;
        ++item_local;
      }
      if (issued) {
        // all MMAs of this CTA complete before TMEM is released
        tc_commit(&bars.teardown);
        mbar_wait(&bars.teardown, 0, nullptr, &g_sol_status, 0, lim);
      }
    }
    __syncwarp();
  } else {
    // ================================================================ softmax + epilogue
    const int quad = warp & 3;           // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;    // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t g = 0;
    int item_local = 0;
    bool ok = true;
    for (int it = 0;; ++it) {
      const int slot = it & 1;
      if (!(ok = wait_bar_warp(&bars.item_full[slot], (it >> 1) & 1, bars, lim, 20))) break;
      const int item = bars.item_slot[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
      if (item < 0) break;
      const int bh = item / p.N, qi = item % p.N;
      const int T = p.tiles[item];
      const int n_rows = min(BM, p.L - qi * BM);
      __nv_bfloat16* orow = p.out + ((size_t)bh * p.L + (size_t)qi * BM + row) * HD;
      if (T == 0) {
        if (row < n_rows)
          for (int c = 0; c < HD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      TileIter ti;
      ti.init(p.mask + (size_t)item * p.W, p.W, p.N, p.nchunk);
      float m_used = -INFINITY, l = 0.f;
      for (int n = 0; n < T; ++n) {
        int kind = 0, tidx = 0;
        ti.next(kind, tidx);
        const uint32_t gs = g + n;
        const int sb = gs & 1;
        if (!(ok = wait_bar_warp(&bars.s_full[sb], (gs >> 1) & 1, bars, lim, 21))) break;
        tc_fence_after();
        float x[128];
        {
          uint32_t r[32];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tmem_ld32(tmem + lane_off + TM_S + sb * 128 + q * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) x[q * 32 + c] = __uint_as_float(r[c]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.s_free[sb]);

        // column validity and bias of this tile
        float rmax;
        if (kind == 1 && (tidx != p.N - 1 || p.n_last == BN)) {
          const uint32_t vm[4] = {~0u, ~0u, ~0u, ~0u};
          rmax = tile_logits<true>(x, p.scale_log2, 0.f, vm, -1, 0.f);
        } else {
          uint32_t vm[4];
          float bias = 0.f;
          int sc = -1;
          float sc_delta = 0.f;
          if (kind == 1) {  // partial last key block: columns >= n_last are padding
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int nb = p.n_last - q * 32;
              vm[q] = nb >= 32 ? ~0u : (nb <= 0 ? 0u : ((1u << nb) - 1u));
            }
          } else {  // pooled chunk: unselected, in-range blocks only
            bias = p.bias_full;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int w = tidx * 4 + q;
              vm[q] = (w < p.W) ? ((~p.mask[(size_t)item * p.W + w]) & ti.valid_bits(w)) : 0u;
            }
            const int jl = p.N - 1 - tidx * BN;
            if (jl >= 0 && jl < BN && p.n_last != BN) {
              sc = jl;
              sc_delta = p.bias_last - p.bias_full;
            }
          }
          rmax = tile_logits<false>(x, p.scale_log2, bias, vm, sc, sc_delta);
        }
        const float m_new = fmaxf(m_used, rmax);
        const bool need = m_new > m_used + RESCALE_THRESHOLD;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
          l *= alpha;
        }
        uint32_t pk[2][32];
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float p0 = ex2_approx(x[c] - m_used);
          const float p1 = ex2_approx(x[c + 1] - m_used);
          rs += p0 + p1;
          pk[c >> 6][(c & 63) >> 1] = pack_bf16x2(p0, p1);
        }
        l += rs;
        // P buffer sb was read by the PV of tile gs - 2
        if (gs >= 2 && !(ok = wait_bar_warp(&bars.pv_done[sb], ((gs - 2) >> 1) & 1, bars, lim, 22))) break;
        tmem_st32(tmem + lane_off + TM_P + sb * 64, pk[0]);
        tmem_st32(tmem + lane_off + TM_P + sb * 64 + 32, pk[1]);
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          // O must hold every PV up to tile gs - 1 before it is rescaled
          const uint32_t gp = gs - 1;
          if (!(ok = wait_bar_warp(&bars.pv_done[gp & 1], (gp >> 1) & 1, bars, lim, 23))) break;
          tc_fence_after();
          uint32_t o[32];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tmem_ld32(tmem + lane_off + TM_O + q * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tmem + lane_off + TM_O + q * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[sb]);
      }
      if (!ok) break;
      // epilogue: O / l for this row
      if (!(ok = wait_bar_warp(&bars.o_full, item_local & 1, bars, lim, 24))) break;
      tc_fence_after();
      const float inv = 1.0f / l;
      uint32_t ob[4][32];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld32(tmem + lane_off + TM_O + q * 32, ob[q]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_free);
      if (row < n_rows) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ob[q][c + 0]) * inv, __uint_as_float(ob[q][c + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ob[q][c + 2]) * inv, __uint_as_float(ob[q][c + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ob[q][c + 4]) * inv, __uint_as_float(ob[q][c + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ob[q][c + 6]) * inv, __uint_as_float(ob[q][c + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + q * 32 + c) = w;
          }
        }
      }
      g += T;
      ++item_local;
    }
    // an abandoned tile may leave a TMEM access in flight
    tmem_wait_ld();
    tmem_wait_st();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// [planes, rows, 128] bf16 tensor, boxes of 64 columns x 128 rows, 128-byte
// swizzle; rows past `rows` read as zero.
bool make_map(CUtensorMap* m, const void* base, int rows, int planes) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)rows * HD * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* out, const Geometry& g,
                           const Scratch& s, cudaStream_t st, uint64_t wait_limit_ns) {
  CUtensorMap mQ, mK, mV, mKb, mVb;
  if (!make_map(&mQ, q, g.L, g.bH) || !make_map(&mK, k, g.L, g.bH) || !make_map(&mV, v, g.L, g.bH) ||
      !make_map(&mKb, s.kbar_op, g.N, g.bH) || !make_map(&mVb, s.vbar_op, g.N, g.bH))
    return cudaErrorInvalidValue;
  Params p;
  p.bH = g.bH; p.L = g.L; p.N = g.N; p.W = g.W; p.nchunk = g.nchunk; p.nitems = g.nitems; p.n_last = g.n_last;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
  p.bias_full = (float)std::log2((double)g.B);
  p.bias_last = (float)std::log2((double)g.n_last);
  p.mask = s.mask; p.tiles = s.tiles; p.order = s.order; p.work_counter = s.work_counter;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.wait_limit_ns = wait_limit_ns;
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = g.nitems < nsm ? g.nitems : nsm;
  attn_tc_kernel<<<grid, NTHREADS, SMEM_BYTES, st>>>(mQ, mK, mV, mKb, mVb, p);
  return cudaGetLastError();
}

cudaError_t read_device_status(cudaStream_t st, int32_t* word) {
  int32_t w = 0;
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(&w, g_sol_status, sizeof(w));
  if (e != cudaSuccess) return e;
  const int32_t zero = 0;
  e = cudaMemcpyToSymbol(g_sol_status, &zero, sizeof(zero));
  if (word) *word = w;
  return e;
}

}  // namespace sol
