// attn_tc.cu -- the Sol-Attn attention loop on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), bf16 operands, fp32 accumulation, d = 128 or 64,
// query blocks of 128 or 64 tokens, key blocks of 128 or 64 tokens.
//
// What sets the pace is the softmax of each tile and the round trip it
// waits on: P of tile n is written over S in TMEM, so S of tile n + 2 can be
// computed only after PV of tile n, and the softmax of a tile (max, 64
// exponentials per thread, the bf16 P) is about as long as the tile's
// tensor work.  The control warps are kept lean (descriptors built once, one
// commit per MMA group, the selection row in registers, waits that probe
// before they block), most exponentials go to the MUFU unit, and the merge
// and store of each query block's output is left to a separate warpgroup.
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
//     Only selected K/V tiles are ever loaded.  With 64-token key blocks one
//     128-column tile holds two selected blocks, one per softmax column half
//     (an odd count leaves the last tile's second half masked out).
//   With 64-token query blocks one 128-row tile holds two blocks (rows 0-63
//   and 64-127): the tile sequence is the union of their selections, and each
//   row half masks out what its own block takes through the other path.
//
// Persistent CTAs, one per SM, 512 threads in four warpgroups (every
// scheduler hosts one warp of each; the registers are rebalanced at start
// with setmaxnreg: 72 per thread for the control warpgroup, 176 for the
// softmax, 88 for the epilogue):
//   warp 0        TMA producer: fetches work items, loads the Q tile and each
//                 tile's K and V (or K-bar and V-bar) together into a 3-stage
//                 ring (6 at d = 64)
//   warp 1        TMEM owner and tcgen05.mma issuer (one elected lane)
//   warps 2, 3    in-kernel routing only: fetch the work items and decide
//                 each one's selection ahead of the producer (half the
//                 pooled-key chunks each)
//   warps 4..11   softmax, two column halves: half h owns the 64 keys
//                 [64h, 64h + 64) of every tile, one query row per thread (its
//                 warp's TMEM lane quadrant).  Each half keeps its own running
//                 max, row sum and fp32 accumulator O_h = sum P_h V_h, so the
//                 halves never wait for each other inside the key loop; at the
//                 end of a query block they leave their row states in shared
//                 memory and go on with the next block.
//   warps 12..15  epilogue: merge the two partial softmax states of each row
//                 and write the output row (bf16), one row per thread.
// TMEM columns: two S buffers [0,128) and [128,256) (tile n in buffer n % 2,
// so S of the next tile is computed while the softmax works on this one; the
// softmax writes P as bf16 pairs over the first 32 columns of each 64-column
// half of its S), O_0 [256,384), O_1 [384,512).  At d = 64 an accumulator
// takes 64 columns, so consecutive query blocks alternate between two banks
// (O_h of bank b at 256 + 128 h + 64 b).
// Every mbarrier wait is bounded; on expiry the CTA abandons its work, waits
// for its own copies and MMAs, frees TMEM and records the failing wait in the
// device status word.
#include <cmath>
#include <cstddef>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace sol {

__device__ int g_sol_status;  // 0 = ok; else 0x1000 | wait id (first expiry), 0x3000 | check id

// Per-CTA record of the last attention launch on this device (a measurement
// aid for load balance): start and end time (%globaltimer, ns), work items
// and tiles the CTA processed.  Two timer reads and four stores per CTA.
__device__ unsigned long long g_cta_times[kMaxCtaTimes][4];

// Consistency checks of the debug build (-DSOL_ATTN_DEBUG_CHECKS): a failed
// check records its id in the status word (first failure wins) instead of
// trapping, and the kernel carries on; the release build compiles them away.
#ifdef SOL_ATTN_DEBUG_CHECKS
#define SOL_DCHECK(cond, id)                                     \
  do {                                                           \
    if (!(cond)) atomicCAS(&g_sol_status, 0, 0x3000 | (id));     \
  } while (0)
#else
#define SOL_DCHECK(cond, id) \
  do {                       \
  } while (0)
#endif

namespace {

constexpr int BM = 128, BN = 128;
constexpr int QST = 1;  // Q buffers
// 16 warps in four warpgroups: control (producer, MMA, router, idle),
// two softmax warpgroups (one per column half) and the epilogue warpgroup.
// Warp w may access TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, so every
// warpgroup covers the four lane quadrants, and every scheduler (w % 4) hosts
// one warp of each warpgroup.
constexpr int NTHREADS = 512;
constexpr int ROUTER_WARP = 2;  // in-kernel routing: warps 2 and 3 score the items ahead of the producer
constexpr int SOFTMAX_WARPS = 8;
constexpr int SOFTMAX_WARP0 = 4;  // warps 4..11: half (w - 4) / 4, quadrant w % 4
constexpr int EPI_WARP0 = 12;     // warps 12..15: the epilogue, quadrant w % 4
constexpr int EPI_WARPS = 4;
// registers per thread after the warpgroups rebalance (setmaxnreg), within
// the 64 K of the SM: 128 x 72 + 256 x 176 + 128 x 88 = 65536
constexpr int REG_CONTROL = 72, REG_SOFTMAX = 176, REG_EPI = 88;
static_assert(128 * REG_CONTROL + 256 * REG_SOFTMAX + 128 * REG_EPI <= 65536, "register split");
constexpr uint32_t SLAB = BM * 128;  // 16 KB: 64 bf16 columns of a 128-row tile, 128-byte swizzled

// Shared-memory plan for head dimension HD (64 or 128).  A Q, K or V tile is
// HD / 64 slabs; the K+V ring gets as many stages as fit (3 at d = 128, 6 at
// d = 64).  There is no room for alignment slack: the kernel checks that
// dynamic shared memory starts on a 1024-byte boundary (the 128-byte swizzle
// needs it) and reports an error instead of running if it does not.
template <int HD>
struct Cfg {
  static_assert(HD == 64 || HD == 128, "head dimension");
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t TILE_BYTES = NSLAB * SLAB;
  static constexpr int KVST = HD == 128 ? 3 : 6;  // K+V stages
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_KV = OFF_Q + QST * TILE_BYTES;  // stage s: K at +2s tiles, V at +2s+1
  static constexpr uint32_t OFF_BAR = OFF_KV + 2 * KVST * TILE_BYTES;
  // barriers, tile descriptors and row states: 3 KB fill the last of the
  // 227 KB at d = 128; d = 64 leaves room for its six descriptors
  static constexpr uint32_t BAR_AREA = HD == 128 ? 3072 : 4096;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_AREA;
};
static_assert(Cfg<128>::SMEM_BYTES <= 227 * 1024 && Cfg<64>::SMEM_BYTES <= 227 * 1024, "shared memory");

// TMEM columns: S buffer b at TM_S + 128 b (tile gs uses buffer gs % 2; its
// P overwrites the first 32 columns of each 64-column half, as bf16 pairs),
// O_h at TM_O + 128 h
constexpr uint32_t TM_S = 0, TM_O = 256;
// O banks: at d = 64 an accumulator takes 64 of its half's 128 columns, so
// consecutive items alternate between two banks and an item's PVs need not
// wait for the previous item's epilogue to read O
template <int HD>
constexpr int o_banks() { return HD == 64 ? 2 : 1; }
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

// A share of the probabilities goes through an FMA-pipe polynomial exp2
// instead of the MUFU ex2 unit: npoly<HD>() of every 8 column pairs.  At
// d = 128 the softmax warps are bound by issue slots rather than by MUFU
// throughput (4 lanes per cycle per scheduler), and the polynomial costs five
// times the issue slots of MUFU: measured on Wan 720p, 0 to 4 of 8 lie within
// the clock spread, 1 of 8 is kept.  At d = 64 a tile's tensor work halves
// while its exponentials stay, MUFU sets the pace, and 3 of 8 measured fastest
// (image-DiT d = 64, beta = 1.04: 0.325 of the measured peak against 0.310).
template <int HD>
constexpr int npoly() { return HD == 64 ? 3 : 1; }
template <int NP>
__host__ __device__ constexpr bool poly_pair(int pair) {
  return NP >= 3   ? ((pair & 7) == 2 || (pair & 7) == 5 || (pair & 7) == 7)
         : NP == 2 ? ((pair & 7) == 3 || (pair & 7) == 7)
         : NP == 1 ? (pair & 7) == 7
                   : false;
}

struct Params {
  int bH, L, Nq, Nk, W, nchunk, nitems, nk_last;
  int pair;             // 1: key blocks of 64 tokens, two per exact tile; 0: blocks of 128
  // 1: query blocks of 64 tokens, two per 128-row tile: item t of head bh is
  // the pair of query blocks 2t and 2t + 1 (rows [128 t, 128 t + 128)), which
  // walks the union of their selections (items taken heaviest first by the
  // sum of the two blocks' tile counts); 0: query blocks of 128 tokens
  int rowpair;
  int Ni;               // items per head: Nq, or ceil(Nq / 2) with rowpair
  float scale_log2;     // log2(e) / sqrt(d)
  float bias_full;      // log2(Bk)
  float bias_last;      // log2(nk_last)
  const uint32_t* mask;
  const int32_t* tiles;
  const int32_t* order;
  int32_t* work_counter;
  __nv_bfloat16* out;
  uint64_t wait_limit_ns;
  int chunks;           // pooled-key chunks walked per item: nchunk, or 0 without the correction
  // routing inside the kernel (route_inkernel != 0): the producer warp decides
  // S_i from the fp32 pooled vectors and the router's tau_i instead of reading
  // the mask; the arithmetic is the router's, so the sets are identical
  int route_inkernel;
  int test_stall;       // failure-detection tests: the CTA's first S is never signalled
  int out_align32;      // the output is 32-byte aligned: rows are written with 32-byte stores
  float scale;          // 1/sqrt(d) as the router computes it
  const float* qbar;    // [bH, Nq, d] fp32
  const float* kbar;    // [bH, Nk, d] fp32
  const float* tau;     // [bH * Nq]
};

// What the producer tells the other roles about the tile in one ring stage:
// kind 0 = pooled chunk idx (vm[r]: the unselected, in-range pooled keys of
// row half r's query block, 4 words), kind 1 = exact key block idx (and idx2
// for a 64-token pair, or -1); sel bit 2 c + r: the tile's c-th key block is
// selected by row half r's query block.  With 128-token query blocks both row
// halves hold the same block.
struct TileDesc {
  int kind, idx, idx2, sel;
  uint32_t vm[2][4];
};

template <int KVST>
struct Bars {
  uint64_t q_full[QST], q_empty[QST];
  uint64_t kv_full[KVST], kv_empty[KVST];
  uint64_t s_full[2];     // [S buffer]: S of the buffer's tile is in TMEM
  uint64_t p_full[2];     // [S buffer]: both column halves have written P over S
  uint64_t o_full[2], o_free[2];  // [O bank]: the item's last PV is done / the epilogue has read O
  uint64_t item_full[2], item_empty[2];
  uint64_t state_full;     // the softmax warps have left the item's row states
  uint64_t state_empty;    // the epilogue has read them
  uint64_t teardown;
  int item_slot[2];
  int item_T[2];          // tiles of the item in each slot
  TileDesc desc[KVST];    // per ring stage, written before the stage's loads are armed
  // in-kernel routing: the router warp hands each item (index, tile count,
  // selection words) to the producer through two slots
  uint64_t rq_full[2], rq_empty[2];
  int rq_item[2], rq_T[2];
  uint32_t rq_bits[2][64];
  int rr_item;            // the item the two router warps score next (router warp 0 fetches it)
  int rr_part[2];         // router warp 1's selected-block and chunk counts
  uint32_t tmem_base;
  int abort_flag;
  float xm[2][BM];        // [column half][row] running max (log2 units)
  float xl[2][BM];        // [column half][row] row sum
};
static_assert(sizeof(Bars<Cfg<64>::KVST>) <= Cfg<64>::BAR_AREA && sizeof(Bars<Cfg<128>::KVST>) <= Cfg<128>::BAR_AREA,
              "barrier area");
static_assert(QST == 1, "one Q buffer");

// Walks the tile sequence of one work item: pooled-key chunks holding an
// unselected block, then the selected blocks in increasing order (one per
// tile, or two with 64-token key blocks).  An item of two 64-token query
// blocks walks the union: a key block is exact if either block selected it,
// and a chunk is walked if it holds a block that either left unselected.
// The selection words come from the router's mask rows in global memory, or
// (m == nullptr) from registers of the warp: lane (w % 32) holds word w in
// rb0 / rc0 (w < 32) or rb1 / rc1.  Every lane of the warp runs the same calls.
struct TileIter {
  const uint32_t* m;   // row of the (first) query block
  const uint32_t* m2;  // row of the second query block (two == true)
  uint32_t rb0, rb1, rc0, rc1;
  bool two;
  int W, N, nchunk, pair;
  int chunk;     // next chunk to test
  int word;      // current mask word in the exact phase
  uint32_t bits; // remaining set bits of that word
  __device__ void init(const uint32_t* mrow, int W_, int N_, int nchunk_, int pair_) {
    m = mrow; m2 = mrow; rb0 = rb1 = rc0 = rc1 = 0; two = false; W = W_; N = N_; nchunk = nchunk_; pair = pair_;
    chunk = 0; word = -1; bits = 0;
  }
  // mask word w of the first and the second query block (the same word for one block)
  __device__ __forceinline__ void load_words(int w, uint32_t& a, uint32_t& b) const {
    if (m) {
      a = m[w];
      b = two ? m2[w] : a;
    } else {
      a = __shfl_sync(0xffffffffu, w < 32 ? rb0 : rb1, w & 31);
      b = two ? __shfl_sync(0xffffffffu, w < 32 ? rc0 : rc1, w & 31) : a;
    }
  }
  // blocks of mask word w left unselected (and in range) by the first / the second block
  __device__ __forceinline__ void unselected2(int w, uint32_t& ua, uint32_t& ub) const {
    if (w >= W) { ua = ub = 0u; return; }
    uint32_t a, b;
    load_words(w, a, b);
    const uint32_t v = valid_bits(w);
    ua = ~a & v;
    ub = ~b & v;
  }
  // 2 bits: key block j is selected by the first (bit 0) / the second (bit 1) block
  __device__ __forceinline__ int sel_bits(int j) const {
    uint32_t a, b;
    load_words(j >> 5, a, b);
    return (int)((a >> (j & 31)) & 1u) | (int)(((b >> (j & 31)) & 1u) << 1);
  }
  __device__ __forceinline__ int next_selected() {
    while (bits == 0) {
      if (++word >= W) return -1;
      uint32_t a, b;
      load_words(word, a, b);
      bits = a | b;
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1;
    return word * 32 + b;
  }
  __device__ __forceinline__ uint32_t valid_bits(int w) const {
    const int nb = N - w * 32;
    return nb >= 32 ? 0xffffffffu : (nb <= 0 ? 0u : ((1u << nb) - 1u));
  }
  // kind 0: pooled chunk idx; kind 1: exact key block idx (and, in pair mode,
  // idx2 = the second block of the tile or -1).  false when done.
  __device__ bool next(int& kind, int& idx, int& idx2) {
    idx2 = -1;
    while (chunk < nchunk) {
      const int c = chunk++;
      uint32_t un = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t ua, ub;
        unselected2(c * 4 + q, ua, ub);
        un |= ua | ub;
      }
      if (un) { kind = 0; idx = c; return true; }
    }
    idx = next_selected();
    if (idx < 0) return false;
    if (pair) idx2 = next_selected();
    kind = 1;
    return true;
  }
};

// Eq. 4 decided inside the kernel for query block `item`, over the chunks of
// 128 pooled keys c = c0, c0 + cstep, ...: the whole warp forms
// s_ij = (Q-bar_i . K-bar_j) / sqrt(d) for the chunk's key blocks j, four per
// lane at a time, with the router's arithmetic (fp32, one fused multiply-add
// per channel in channel order, then the scale), and writes the bits j with
// s_ij > tau_i as the chunk's mask words into bits (shared memory).  Q-bar_i
// is read with broadcast loads (every lane the same address).  Adds to cnt the
// selected blocks and to used the chunks holding an unselected block.
template <int HD>
__device__ void route_part(const Params& p, int item, int lane, int c0, int cstep, uint32_t* bits, int& cnt,
                           int& used) {
  const int bh = item / p.Nq;
  SOL_DCHECK(p.W <= 64, 7);
  const float4* qrow = reinterpret_cast<const float4*>(p.qbar + (size_t)item * HD);
  const float tau = __ldg(p.tau + item);
  const float* kb = p.kbar + (size_t)bh * p.Nk * HD;
  const int nch = (p.Nk + 127) >> 7;
  for (int c = c0; c < nch; c += cstep) {
    float acc[4];
    const float* kr[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = c * 128 + r * 32 + lane;
      kr[r] = kb + (size_t)(j < p.Nk ? j : 0) * HD;  // rows past Nk read row 0 and are masked below
      acc[r] = 0.f;
    }
#pragma unroll 4
    for (int cc = 0; cc < HD; cc += 4) {
      const float4 q4 = __ldg(qrow + (cc >> 2));
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 k4 = __ldg(reinterpret_cast<const float4*>(kr[r] + cc));
        acc[r] = fmaf(q4.x, k4.x, acc[r]);
        acc[r] = fmaf(q4.y, k4.y, acc[r]);
        acc[r] = fmaf(q4.z, k4.z, acc[r]);
        acc[r] = fmaf(q4.w, k4.w, acc[r]);
      }
    }
    bool any_unselected = false;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int w = c * 4 + r;  // keys 32w .. 32w + 31
      const bool bit = (32 * w + lane < p.Nk) && (acc[r] * p.scale > tau);
      const uint32_t word = __ballot_sync(0xffffffffu, bit);
      if (w < p.W) {
        if (lane == 0) bits[w] = word;
        cnt += __popc(word);
        const int nb = p.Nk - w * 32;
        const uint32_t valid = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
        any_unselected |= ((~word) & valid) != 0u;
      }
    }
    used += any_unselected ? 1 : 0;
  }
}

// Named barrier of the two router warps (warps 2 and 3, 64 threads).
__device__ __forceinline__ void router_bar() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

// All 32 lanes wait; the outcome is made warp-uniform so that warp-wide
// instructions that follow are never reached by part of a warp.
template <class BarsT>
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, BarsT& B_, uint64_t lim, int id) {
  const bool ok = mbar_wait(bar, parity, &B_.abort_flag, &g_sol_status, 0x1000 | id, lim);
  return __all_sync(0xffffffffu, ok);
}

// 2^x for x <= 8 on the FMA pipe: x = j + f with j = round(x), f in [-1/2, 1/2];
// 2^f from a cubic fitted here to 2^f on [-1/2, 1/2] (least squares with
// Lawson reweighting toward minimax relative error, max 7.5e-5), then j is
// added to the exponent field.  Inputs below -125 (where the exponent field
// would underflow, -inf included) give 2^-125, about 2.4e-38: against row
// sums of at least 1 that is below float precision, so no select is spent on
// returning an exact 0.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 xc = make_float2(fmaxf(x.x, -125.0f), fmaxf(x.y, -125.0f));
  const float shifter = 12582912.0f;  // 1.5 * 2^23: xc + shifter rounds xc to an integer in the low bits
  const float2 t = add2(xc, make_float2(shifter, shifter));
  const float2 j = add2(t, make_float2(-shifter, -shifter));
  const float2 f = add2(xc, make_float2(-j.x, -j.y));
  float2 p = fma2(make_float2(0.05517118f, 0.05517118f), f, make_float2(0.24261113f, 0.24261113f));
  p = fma2(p, f, make_float2(0.69326109f, 0.69326109f));
  p = fma2(p, f, make_float2(0.99992806f, 0.99992806f));
  // the low bits of t hold j; shifting them into the exponent field adds j to p's exponent
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// 2^(x sl2v + negv) of 64 scores as bf16 pairs into pk; returns the sum of
// the (unrounded) probabilities.
template <int NP>
__device__ __forceinline__ float exp_pack64(const float (&x)[64], float2 sl2v, float2 negv, uint32_t (&pk)[32]) {
  float2 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    const float2 a = fma2(make_float2(x[c], x[c + 1]), sl2v, negv);
    float2 e;
    if (poly_pair<NP>(c >> 1)) {
      e = exp2_poly2(a);
    } else {
      e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
    }
    acc[(c >> 1) & 3] = add2(acc[(c >> 1) & 3], e);
    pk[c >> 1] = pack_bf16x2(e.x, e.y);
  }
  const float2 s2 = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  return s2.x + s2.y;
}

// Max of 64 values with three-input max instructions.
__device__ __forceinline__ float tree_max64(const float (&x)[64]) {
  float a[22];
#pragma unroll
  for (int i = 0; i < 21; ++i) a[i] = max3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
  a[21] = x[63];
  float b[8];
#pragma unroll
  for (int i = 0; i < 7; ++i) b[i] = max3(a[3 * i], a[3 * i + 1], a[3 * i + 2]);
  b[7] = a[21];
  return max3(max3(b[0], b[1], b[2]), max3(b[3], b[4], b[5]), fmaxf(b[6], b[7]));
}

template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                   const __grid_constant__ CUtensorMap tmVb, const Params p) {
  using C = Cfg<HD>;
  constexpr int KVST = C::KVST;
  constexpr int NSLAB = C::NSLAB;
  constexpr uint32_t TILE_BYTES = C::TILE_BYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(&g_sol_status, 0, 0x2000);
    return;
  }
  uint8_t* smem = smem_raw;
  Bars<KVST>& bars = *reinterpret_cast<Bars<KVST>*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QST; ++s) { mbar_init(&bars.q_full[s], 1); mbar_init(&bars.q_empty[s], 1); }
    for (int s = 0; s < KVST; ++s) { mbar_init(&bars.kv_full[s], 1); mbar_init(&bars.kv_empty[s], 1); }
    mbar_init(&bars.s_full[0], 1);
    mbar_init(&bars.s_full[1], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.p_full[s], SOFTMAX_WARPS);
      mbar_init(&bars.item_full[s], 1);
      mbar_init(&bars.item_empty[s], 1 + SOFTMAX_WARPS + EPI_WARPS);
      mbar_init(&bars.o_full[s], 1);
      mbar_init(&bars.o_free[s], EPI_WARPS);
    }
    mbar_init(&bars.state_full, SOFTMAX_WARPS);
    mbar_init(&bars.state_empty, EPI_WARPS);
    mbar_init(&bars.teardown, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(&bars.rq_full[s], 1); mbar_init(&bars.rq_empty[s], 1); }
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
  const unsigned long long t_start = globaltimer_ns();
  int n_items_done = 0, n_tiles_done = 0;  // producer's count, for the per-CTA record

  if (warp < 4) {
    setmaxnreg_dec<REG_CONTROL>();
    if (warp == 0) {
      // ================================================================ producer (whole warp, one lane issues)
      const bool leader = elect_one();
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t g = 0;          // global tile counter
      // last K / V tile and number of Q tiles whose loads were issued (to let
      // them land if the CTA abandons its work)
      int gk_last = -1, q_uses = 0;
      bool ok = true;
      for (int it = 0;; ++it) {
        const int slot = it & 1;
        if (it >= 2 && !(ok = wait_warp(&bars.item_empty[slot], ((it >> 1) + 1) & 1, bars, lim, 1))) break;
        int item = -1, T = 0;
        TileIter ti;
        if (p.route_inkernel) {
          // the router warp has fetched and scored the item already
          if (!(ok = wait_warp(&bars.rq_full[slot], (it >> 1) & 1, bars, lim, 4))) break;
          item = bars.rq_item[slot];
          T = bars.rq_T[slot];
          ti.init(bars.rq_bits[slot], p.W, p.Nk, p.chunks, p.pair);
        } else {
          int idx = 0;
          if (lane == 0) idx = atomicAdd(p.work_counter, 1);
          idx = __shfl_sync(0xffffffffu, idx, 0);
          item = idx < p.nitems ? p.order[idx] : -1;
          if (item >= 0) {
            // mask row of the item's (first) query block, and of the second
            // one of a pair when it exists
            const int blk = p.rowpair ? (item / p.Ni) * p.Nq + 2 * (item % p.Ni) : item;
            const uint32_t* mrow = p.mask + (size_t)blk * p.W;
            const bool two = p.rowpair && 2 * (item % p.Ni) + 1 < p.Nq;
            if (p.W <= 64) {
              // the item's selection row in two registers per lane (one
              // coalesced load): walking its tiles then costs shuffles, not a
              // dependent L2 round trip per mask word
              ti.init(nullptr, p.W, p.Nk, p.chunks, p.pair);
              ti.rb0 = lane < p.W ? __ldg(mrow + lane) : 0u;
              ti.rb1 = 32 + lane < p.W ? __ldg(mrow + 32 + lane) : 0u;
              if (two) {
                ti.rc0 = lane < p.W ? __ldg(mrow + p.W + lane) : 0u;
                ti.rc1 = 32 + lane < p.W ? __ldg(mrow + p.W + 32 + lane) : 0u;
              }
            } else {
              ti.init(mrow, p.W, p.Nk, p.chunks, p.pair);
              ti.m2 = mrow + p.W;
            }
            ti.two = two;
            if (p.rowpair && p.W <= 64) {
              // the union's tile count from the rows in registers: selected
              // blocks of either query block, and the chunks (4 words each)
              // holding a block that either left unselected
              const uint32_t a0 = ti.rb0, a1 = ti.rb1;
              const uint32_t b0 = two ? ti.rc0 : a0, b1 = two ? ti.rc1 : a1;
              const int cnt = __reduce_add_sync(0xffffffffu, __popc(a0 | b0) + __popc(a1 | b1));
              const uint32_t f0 = __ballot_sync(0xffffffffu, lane < p.W && (~(a0 & b0) & ti.valid_bits(lane)) != 0u);
              const uint32_t f1 =
                  __ballot_sync(0xffffffffu, 32 + lane < p.W && (~(a1 & b1) & ti.valid_bits(32 + lane)) != 0u);
              int used = 0;
              for (int c = 0; c < p.chunks; ++c) used += (((c < 8 ? f0 >> (4 * c) : f1 >> (4 * (c - 8))) & 0xfu) != 0u);
              T = used + (p.pair ? (cnt + 1) >> 1 : cnt);
            } else if (p.rowpair) {
              // the union's tile count: one walk of a copy of the iterator
              TileIter tc = ti;
              int kd, i1, i2;
              T = 0;
              while (tc.next(kd, i1, i2)) ++T;
            } else {
              T = p.tiles[item];
            }
          }
        }
        if (lane == 0) {
          bars.item_slot[slot] = item;
          bars.item_T[slot] = T;
          mbar_arrive(&bars.item_full[slot]);
        }
        if (item < 0) break;
        const int bh = item / p.Ni, qi = item % p.Ni;  // qi: the item's 128-row tile of Q
        SOL_DCHECK(item < p.nitems && bh < p.bH && T >= 0, 1);
        // the router's slot is released once this item's selection words are no
        // longer read (after its last tile is issued)
        auto release_route_slot = [&]() {
          if (p.route_inkernel && lane == 0) mbar_arrive(&bars.rq_empty[slot]);
        };
        if (T == 0) {
          release_route_slot();
          ++n_items_done;
          continue;
        }
        // Q tile into buffer q_uses % QST, once the item that used it last has
        // issued all its S MMAs
        const int qb = q_uses % QST;
        const int qu = q_uses / QST;
        if (qu > 0 && !(ok = wait_warp(&bars.q_empty[qb], (qu - 1) & 1, bars, lim, 2))) break;
        if (leader) {
          mbar_arrive_expect_tx(&bars.q_full[qb], TILE_BYTES);
          uint8_t* qdst = smem + C::OFF_Q + qb * TILE_BYTES;
  #pragma unroll
          for (int hd = 0; hd < NSLAB; ++hd)
            tma_load_3d(qdst + hd * SLAB, &tmQ, &bars.q_full[qb], hd * 64, qi * BM, bh, pol_q);
        }
        ++q_uses;
        for (int n = 0; n < T; ++n) {
          int kind = 0, tidx = 0, tidx2 = -1;
          const bool has_tile = ti.next(kind, tidx, tidx2);
          SOL_DCHECK(has_tile, 2);  // the item's tile count matches its selection
          SOL_DCHECK(kind == 1 ? (tidx >= 0 && tidx < p.Nk && tidx2 < p.Nk && (p.pair || tidx2 < 0))
                               : (tidx >= 0 && tidx < p.chunks),
                     3);
          uint32_t vm[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
          int sel = 0;
          if (kind == 0) {
  #pragma unroll
            for (int q = 0; q < 4; ++q) ti.unselected2(tidx * 4 + q, vm[0][q], vm[1][q]);
          } else {
            sel = !p.rowpair ? 0xf : (ti.sel_bits(tidx) | (tidx2 >= 0 ? ti.sel_bits(tidx2) << 2 : 0));
          }
          const uint32_t gk = g + n;
          const int ks = gk % KVST;
          const int ku = gk / KVST;
          // stage ks is free once the PV of its previous tile has finished
          if (ku > 0 && !(ok = wait_warp(&bars.kv_empty[ks], (ku - 1) & 1, bars, lim, 3))) break;
          if (leader) {
            uint8_t* dk = smem + C::OFF_KV + (2 * ks) * TILE_BYTES;
            uint8_t* dv = dk + TILE_BYTES;
            TileDesc& td = bars.desc[ks];  // published by the arrive below (release)
            td.kind = kind;
            td.idx = tidx;
            td.idx2 = tidx2;
            td.sel = sel;
  #pragma unroll
            for (int q = 0; q < 4; ++q) {
              td.vm[0][q] = vm[0][q];
              td.vm[1][q] = vm[1][q];
            }
            mbar_arrive_expect_tx(&bars.kv_full[ks], 2 * TILE_BYTES);
            if (kind == 1 && p.pair) {
              // rows [0, 64) <- key block tidx, rows [64, 128) <- key block tidx2;
              // a tile with one block repeats it in the second half (masked out)
              const int j2 = tidx2 >= 0 ? tidx2 : tidx;
  #pragma unroll
              for (int hd = 0; hd < NSLAB; ++hd) {
                tma_load_3d(dk + hd * SLAB, &tmK, &bars.kv_full[ks], hd * 64, tidx * 64, bh, pol_kv);
                tma_load_3d(dk + hd * SLAB + 64 * 128, &tmK, &bars.kv_full[ks], hd * 64, j2 * 64, bh, pol_kv);
                tma_load_3d(dv + hd * SLAB, &tmV, &bars.kv_full[ks], hd * 64, tidx * 64, bh, pol_kv);
                tma_load_3d(dv + hd * SLAB + 64 * 128, &tmV, &bars.kv_full[ks], hd * 64, j2 * 64, bh, pol_kv);
              }
            } else {
              const CUtensorMap* mk = kind ? &tmK : &tmKb;
              const CUtensorMap* mv = kind ? &tmV : &tmVb;
  #pragma unroll
              for (int hd = 0; hd < NSLAB; ++hd) {
                tma_load_3d(dk + hd * SLAB, mk, &bars.kv_full[ks], hd * 64, tidx * BN, bh, pol_kv);
                tma_load_3d(dv + hd * SLAB, mv, &bars.kv_full[ks], hd * 64, tidx * BN, bh, pol_kv);
              }
            }
          }
          gk_last = (int)gk;
        }
        if (!ok) break;
        release_route_slot();
        g += T;
        ++n_items_done;
        n_tiles_done += T;
      }
      if (!ok || bars.abort_flag) {
        // let every copy this warp started land before the CTA exits: the last
        // use of each ring stage is one of the ring's last issued tiles
        for (int back = 0; back < KVST; ++back) {
          const int gk = gk_last - back;
          if (gk >= 0) mbar_wait(&bars.kv_full[gk % KVST], (gk / KVST) & 1, nullptr, &g_sol_status, 0, lim);
        }
        if (q_uses > 0) mbar_wait(&bars.q_full[0], (q_uses - 1) & 1, nullptr, &g_sol_status, 0, lim);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ================================================================ MMA issuer (whole warp, one lane issues)
      const bool leader = elect_one();
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
      // Shared-memory descriptors of the first ring stage and of the Q buffer;
      // a stage or a K-step only moves the start address, the low 14-bit field
      // (address / 16, no carry: shared memory is < 256 KB)
      constexpr uint32_t TILE16 = TILE_BYTES >> 4;
      const uint64_t dK0 = smem_desc_sw128(smem_u32(smem + C::OFF_KV), 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_u32(smem + C::OFF_KV) + TILE_BYTES, SLAB, 1024);
      const uint64_t dQ = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
      static_assert(QST == 1, "one Q descriptor");
      uint32_t g = 0;
      int item_local = 0;  // items with T > 0 processed
      bool issued = false;
      bool ok = true;
      // S_gs = Q K_gs^T into S buffer gs % 2.  The buffer last held tile gs - 2:
      // the softmax read that S before handing over its P, and the PV that read
      // the P was issued before this MMA by this thread, so it is done first.
      // last: this is the item's last S; the Q buffer is released after it.
      auto issue_s = [&](uint32_t gs, bool last, int qb) -> bool {
        const int ks = gs % KVST;
        if (!wait_warp(&bars.kv_full[ks], (gs / KVST) & 1, bars, lim, 15)) return false;
        tc_fence_after();
        if (leader) {
          const uint64_t dK = dK0 + (uint64_t)(2 * ks * TILE16);
          const uint32_t tS = tmem + TM_S + (gs & 1) * 128;
  #pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * SLAB + (kk & 3) * 32) >> 4;
            mma_ss(tS, dQ + off, dK + off, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          if (!(p.test_stall && gs == 0)) tc_commit(&bars.s_full[gs & 1]);
          if (last) tc_commit(&bars.q_empty[qb]);  // every S MMA of this item has been issued
        }
        __syncwarp();
        return true;
      };
      // O_h += P_h V_h for both halves of tile gp (its V arrived with its K),
      // into the item's O bank; the bank's previous item must have been read
      constexpr int NOB = o_banks<HD>();
      auto issue_pv = [&](uint32_t gp, bool first) -> bool {
        const int pb = gp & 1;
        const int ks = gp % KVST;
        const int ob = item_local % NOB;
        if (first && item_local >= NOB &&
            !wait_warp(&bars.o_free[ob], ((item_local / NOB) - 1) & 1, bars, lim, 14))
          return false;
        if (!wait_warp(&bars.p_full[pb], (gp >> 1) & 1, bars, lim, 12)) return false;
        tc_fence_after();
        if (leader) {
          const uint64_t dV = dV0 + (uint64_t)(2 * ks * TILE16);
          const uint32_t tP = tmem + TM_S + pb * 128;
  #pragma unroll
          for (int h = 0; h < 2; ++h) {
  #pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts(tmem + TM_O + h * 128 + ob * 64, tP + h * 64 + kk * 8, dV + ((h * 8192 + kk * 2048) >> 4),
                     IDESC_PV, (first && kk == 0) ? 0u : 1u);
          }
          // frees the tile's stage and tells the softmax that O holds this PV
          tc_commit(&bars.kv_empty[ks]);
        }
        __syncwarp();
        return true;
      };
      for (int it = 0;; ++it) {
        const int slot = it & 1;
        if (!(ok = wait_warp(&bars.item_full[slot], (it >> 1) & 1, bars, lim, 10))) break;
        const int item = bars.item_slot[slot];
        const int T = bars.item_T[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
        if (item < 0) break;
        if (T == 0) continue;
        const int qb = item_local % QST;
        if (!(ok = wait_warp(&bars.q_full[qb], (item_local / QST) & 1, bars, lim, 11))) break;
        // order: S_0, S_1, then for each tile n: PV_n, S_{n+2}
        if (!(ok = issue_s(g, T == 1, qb))) break;
        issued = true;
        if (T > 1 && !(ok = issue_s(g + 1, T == 2, qb))) break;
        for (int n = 0; n < T && ok; ++n) {
          if (!(ok = issue_pv(g + n, n == 0))) break;
          if (n + 2 < T && !(ok = issue_s(g + n + 2, n + 3 == T, qb))) break;
        }
        if (!ok) break;
        if (leader) tc_commit(&bars.o_full[item_local % NOB]);
        __syncwarp();
        g += T;
        ++item_local;
      }
      if (issued) {
        // all MMAs of this CTA complete before TMEM is released
        if (leader) tc_commit(&bars.teardown);
        __syncwarp();
        mbar_wait(&bars.teardown, 0, nullptr, &g_sol_status, 0, lim);
      }
      __syncwarp();
    } else if (warp == ROUTER_WARP || warp == ROUTER_WARP + 1) {
      // ================================================================ router (in-kernel routing only)
      // Two warps on two schedulers share each item's scoring (even and
      // odd chunks of pooled keys), so neither scheduler's softmax warps
      // lose the whole of it.  Router warp 0 fetches the item and hands the
      // result to the producer; the warps meet at two named barriers per
      // item, which both always reach (a failed wait ends the loop through
      // item = -1, not by leaving early).
      const int rw = warp - ROUTER_WARP;
      for (int it = 0; p.route_inkernel; ++it) {
        const int slot = it & 1;
        if (rw == 0) {
          bool ok = true;
          if (it >= 2) ok = wait_warp(&bars.rq_empty[slot], ((it >> 1) + 1) & 1, bars, lim, 5);
          int idx = 0;
          if (lane == 0 && ok) idx = atomicAdd(p.work_counter, 1);
          idx = __shfl_sync(0xffffffffu, idx, 0);
          if (lane == 0) bars.rr_item = ok && idx < p.nitems ? p.order[idx] : -1;
        }
        router_bar();
        const int item = bars.rr_item;
        int cnt = 0, used = 0;
        if (item >= 0) route_part<HD>(p, item, lane, rw, 2, bars.rq_bits[slot], cnt, used);
        if (rw == 1 && lane == 0) {
          bars.rr_part[0] = cnt;
          bars.rr_part[1] = used;
        }
        router_bar();
        if (rw == 0) {
          cnt += bars.rr_part[0];
          used += bars.rr_part[1];
          const int T = item < 0 ? 0 : (p.chunks ? used : 0) + (p.pair ? (cnt + 1) >> 1 : cnt);
          __syncwarp();
          if (lane == 0) {
            bars.rq_item[slot] = item;
            bars.rq_T[slot] = T;
            mbar_arrive(&bars.rq_full[slot]);
          }
        }
        if (item < 0) break;
      }
    }
  } else if (warp >= EPI_WARP0) {
    // ================================================================ epilogue
    // out = (O_0 e_0 + O_1 e_1) / (l_0 e_0 + l_1 e_1), e_h = 2^(m_h - max(m_0, m_1)):
    // the two column halves' partial softmax states of each row, merged once
    // per item while the softmax warps go on with the next item.
    setmaxnreg_dec<REG_EPI>();
    constexpr int NOB = o_banks<HD>();
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int item_local = 0;
    bool ok = true;
    for (int it = 0;; ++it) {
      const int slot = it & 1;
      if (!(ok = wait_warp(&bars.item_full[slot], (it >> 1) & 1, bars, lim, 40))) break;
      const int item = bars.item_slot[slot];
      const int T = bars.item_T[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
      if (item < 0) break;
      const int bh = item / p.Ni, qi = item % p.Ni;  // the item's 128-row tile of Q and of the output
      const int n_rows = min(BM, p.L - qi * BM);
      __nv_bfloat16* orow = p.out + ((size_t)bh * p.L + (size_t)qi * BM + row) * HD;
      if (T == 0) {  // keep-or-drop with nothing selected: the row is 0
        if (row < n_rows)
          for (int c = 0; c < HD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      const int ob = item_local % NOB;
      if (!(ok = wait_warp(&bars.state_full, item_local & 1, bars, lim, 41))) break;
      const float m0 = bars.xm[0][row], m1 = bars.xm[1][row];
      const float l0 = bars.xl[0][row], l1 = bars.xl[1][row];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.state_empty);
      const float mm = fmaxf(m0, m1);
      const float e0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - mm);
      const float e1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - mm);
      // a row whose query block selected nothing without the correction
      // (keep-or-drop; only a pair's second block can meet it here) is 0
      const float den = l0 * e0 + l1 * e1;
      const float inv = den > 0.f ? 1.0f / den : 0.f;
      // every block with tiles has a positive row sum, bar that case
      SOL_DCHECK((inv > 0.f && inv < INFINITY) || (p.rowpair && p.chunks == 0) || row >= n_rows, 6);
      const float w0 = e0 * inv, w1 = e1 * inv;
      if (!(ok = wait_warp(&bars.o_full[ob], (item_local / NOB) & 1, bars, lim, 42))) break;
      tc_fence_after();
      const uint32_t tO0 = tmem + lane_off + TM_O + ob * 64, tO1 = tO0 + 128;
#pragma unroll
      for (int q = 0; q < HD / 32; ++q) {
        uint32_t a[32], b[32];
        tmem_ld32(tO0 + q * 32, a);
        tmem_ld32(tO1 + q * 32, b);
        tmem_wait_ld();
        if (q == HD / 32 - 1) {  // O of this bank read: the MMA may reuse it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.o_free[ob]);
        }
        if (row < n_rows) {
          // one 32-byte store per 16 columns when the output allows it
#pragma unroll
          for (int c = 0; c < 32; c += 16) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w[e] = pack_bf16x2(__uint_as_float(a[c + 2 * e]) * w0 + __uint_as_float(b[c + 2 * e]) * w1,
                                 __uint_as_float(a[c + 2 * e + 1]) * w0 + __uint_as_float(b[c + 2 * e + 1]) * w1);
            if (p.out_align32) {
              st_global_v8(orow + q * 32 + c, w);
            } else {
              *reinterpret_cast<uint4*>(orow + q * 32 + c) = make_uint4(w[0], w[1], w[2], w[3]);
              *reinterpret_cast<uint4*>(orow + q * 32 + c + 8) = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
        }
      }
      ++item_local;
    }
    // an abandoned item may leave a TMEM load in flight
    tmem_wait_ld();
  } else {
    // ================================================================ softmax
    setmaxnreg_inc<REG_SOFTMAX>();
    constexpr int NOB = o_banks<HD>();
    const int half = (warp - SOFTMAX_WARP0) >> 2;  // column half of every S tile this warp owns
    const int quad = warp & 3;            // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;     // query row within the tile
    const int rh = quad >> 1;             // row half: which query block of a 64-token pair
    const int col0 = half * 64;        // this half's key columns of an S tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    int item_local = 0;
    bool ok = true;
    for (int it = 0;; ++it) {
      const int slot = it & 1;
      if (!(ok = wait_warp(&bars.item_full[slot], (it >> 1) & 1, bars, lim, 20))) break;
      const int item = bars.item_slot[slot];
      const int T = bars.item_T[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.item_empty[slot]);
      if (item < 0) break;
      if (T == 0) continue;  // the epilogue writes the zero rows
      // this half's accumulator O_h in the item's O bank
      const uint32_t tO = tmem + lane_off + TM_O + half * 128 + (item_local % NOB) * 64;
      float m_used = -INFINITY, l = 0.f;
      for (int n = 0; n < T; ++n) {
        const uint32_t gs = g + n;
        const int pb = gs & 1;
        const int ks = gs % KVST;
        if (!(ok = wait_warp(&bars.s_full[pb], (gs >> 1) & 1, bars, lim, 21))) break;
        // the tile's descriptor: S_gs being ready implies its stage was filled,
        // and this (already complete) wait orders the producer's writes before
        // the reads; the stage cannot refill before this warp hands over P
        if (!(ok = wait_warp(&bars.kv_full[ks], (gs / KVST) & 1, bars, lim, 22))) break;
        const int kind = bars.desc[ks].kind, tidx = bars.desc[ks].idx, tidx2 = bars.desc[ks].idx2;
        const int tsel = bars.desc[ks].sel;
        SOL_DCHECK((kind == 0 && tidx < p.nchunk) || (kind == 1 && tidx < p.Nk && tidx2 < p.Nk), 4);
        tc_fence_after();
        float x[64];
        {
          uint32_t r0[32], r1[32];
          tmem_ld32(tmem + lane_off + TM_S + pb * 128 + col0, r0);
          tmem_ld32(tmem + lane_off + TM_S + pb * 128 + col0 + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[c] = __uint_as_float(r0[c]);
            x[32 + c] = __uint_as_float(r1[c]);
          }
        }

        // valid key columns of this half of an exact tile: all 64 except in
        // the last (partial) key block and in a pair tile's empty second half
        // (none when this row half's query block did not select the block:
        // it reaches that block through its pooled chunk)
        int nvalid = 64;
        if (kind == 1) {
          if (p.pair) {
            const int jh = half ? tidx2 : tidx;
            nvalid = jh < 0 ? 0 : (jh == p.Nk - 1 ? p.nk_last : 64);
            if (!((tsel >> (2 * half + rh)) & 1)) nvalid = 0;
          } else {
            const int nblk = tidx == p.Nk - 1 ? p.nk_last : BN;
            nvalid = min(max(nblk - col0, 0), 64);
            if (!((tsel >> rh) & 1)) nvalid = 0;
          }
        }
        SOL_DCHECK(nvalid >= 0 && nvalid <= 64, 5);
        // full exact tile: x stays the raw score (scale folded into exp2 below);
        // otherwise x becomes the log2-domain logit with bias and mask applied
        const bool full = kind == 1 && nvalid == 64;
        float lmax;
        if (full) {
          lmax = tree_max64(x) * sl2;  // scaling by sl2 > 0 commutes with max
        } else {
          uint32_t vm[2];
          float bias = 0.f;
          int sc = -1;
          float sc_delta = 0.f;
          if (kind == 1) {  // columns past the valid ones are padding
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int nb = nvalid - q * 32;
              vm[q] = nb >= 32 ? ~0u : (nb <= 0 ? 0u : ((1u << nb) - 1u));
            }
          } else {  // pooled chunk: unselected, in-range blocks only
            bias = p.bias_full;
#pragma unroll
            for (int q = 0; q < 2; ++q) vm[q] = bars.desc[ks].vm[rh][half * 2 + q];
            const int jl = p.Nk - 1 - tidx * BN - col0;
            if (jl >= 0 && jl < 64 && p.bias_last != p.bias_full) {
              sc = jl;
              sc_delta = p.bias_last - p.bias_full;
            }
          }
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            float u = fmaf(x[c], sl2, bias);
            if (c == sc) u += sc_delta;
            x[c] = ((vm[c >> 5] >> (c & 31)) & 1u) ? u : -INFINITY;
          }
          lmax = tree_max64(x);
        }
        // this half's running max (a half may see only masked columns: it
        // then keeps m = -inf and all its probabilities are 0)
        const float m_new = fmaxf(m_used, lmax);
        const bool need = m_new > m_used + RESCALE_THRESHOLD;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
          l *= alpha;
        }
        const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
        const float2 sl2v = make_float2(full ? sl2 : 1.f, full ? sl2 : 1.f);
        const float2 negv = make_float2(neg_m, neg_m);
        uint32_t pk[32];
        l += exp_pack64<npoly<HD>()>(x, sl2v, negv, pk);
        // P over the first 32 columns of this half's S (already in registers).
        // The PV of tile gs - 2 read the previous P of this buffer; it was
        // issued before S of tile gs, and the s_full commit made after that S
        // fires only when all earlier MMAs are done, so no wait is needed
        tmem_st32(tmem + lane_off + TM_S + pb * 128 + col0, pk);
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          // O_h must hold every PV up to tile gs - 1 before it is rescaled
          const uint32_t gp = gs - 1;
          if (!(ok = wait_warp(&bars.kv_empty[gp % KVST], (gp / KVST) & 1, bars, lim, 23))) break;
          tc_fence_after();
#pragma unroll
          for (int q = 0; q < HD / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(tO + q * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + q * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[pb]);
      }
      if (!ok) break;
      // hand this half's softmax state of every row to the epilogue warps
      // (once they have read the previous item's, which they do first)
      if (item_local > 0 && !(ok = wait_warp(&bars.state_empty, (item_local - 1) & 1, bars, lim, 27))) break;
      bars.xm[half][row] = m_used;
      bars.xl[half][row] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.state_full);
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
  if (threadIdx.x == 0 && blockIdx.x < kMaxCtaTimes) {
    unsigned long long* rec = g_cta_times[blockIdx.x];
    rec[0] = t_start;
    rec[1] = globaltimer_ns();
    rec[2] = (unsigned long long)n_items_done;
    rec[3] = (unsigned long long)n_tiles_done;
  }
}


int g_last_grid = 0;  // grid of the last tensor-core attention launch from this process

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

// [planes, rows, HD] bf16 tensor, boxes of 64 columns x box_rows rows,
// 128-byte swizzle; rows past `rows` read as zero.
bool make_map(CUtensorMap* m, const void* base, int HD, int rows, int planes, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)rows * HD * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch_hd(const CUtensorMap& mQ, const CUtensorMap& mK, const CUtensorMap& mV, const CUtensorMap& mKb,
                      const CUtensorMap& mVb, const Params& p, int nitems, cudaStream_t st) {
  constexpr uint32_t smem = Cfg<HD>::SMEM_BYTES;
  int dev = 0, nsm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = nitems < nsm ? nitems : nsm;
  attn_tc_kernel<HD><<<grid, NTHREADS, smem, st>>>(mQ, mK, mV, mKb, mVb, p);
  g_last_grid = grid;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* out, const Geometry& g,
                           const Scratch& s, cudaStream_t st, uint64_t wait_limit_ns, int correction,
                           int route_inkernel, int test_stall) {
  CUtensorMap mQ, mK, mV, mKb, mVb;
  // built for d in {64, 128}, query blocks of 128 tokens (or 64, two to a
  // tile), key blocks of 128 or 64
  if ((g.Bq != BM && g.Bq != BM / 2) || (g.Bk != BN && g.Bk != BN / 2) || (g.d != 64 && g.d != 128))
    return cudaErrorInvalidValue;
  if (!make_map(&mQ, q, g.d, g.L, g.bH, BM) || !make_map(&mK, k, g.d, g.L, g.bH, g.Bk) ||
      !make_map(&mV, v, g.d, g.L, g.bH, g.Bk) || !make_map(&mKb, s.kbar_op, g.d, g.Nk, g.bH, BN) ||
      !make_map(&mVb, s.vbar_op, g.d, g.Nk, g.bH, BN))
    return cudaErrorInvalidValue;
  Params p;
  p.bH = g.bH; p.L = g.L; p.Nq = g.Nq; p.Nk = g.Nk; p.W = g.W; p.nchunk = g.nchunk; p.nitems = g.nitems;
  p.nk_last = g.nk_last;
  p.pair = g.Bk == BN / 2 ? 1 : 0;
  p.rowpair = g.Bq == BM / 2 ? 1 : 0;
  p.Ni = p.rowpair ? (g.Nq + 1) / 2 : g.Nq;
  p.nitems = g.bH * p.Ni;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
  p.bias_full = (float)std::log2((double)g.Bk);
  p.bias_last = (float)std::log2((double)g.nk_last);
  p.mask = s.mask; p.tiles = s.tiles; p.order = s.order; p.work_counter = s.work_counter;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.wait_limit_ns = wait_limit_ns;
  p.chunks = correction ? g.nchunk : 0;
  p.route_inkernel = route_inkernel;
  p.test_stall = test_stall;
  p.out_align32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 ? 1 : 0;
  p.scale = 1.0f / sqrtf((float)g.d);  // the router's expression, evaluated the same way
  p.qbar = s.qbar; p.kbar = s.kbar; p.tau = s.tau;
  if (route_inkernel && (g.W > kInKernelMaxW || !s.tau || p.rowpair)) return cudaErrorInvalidValue;
  if (g.d == 128) return launch_hd<128>(mQ, mK, mV, mKb, mVb, p, p.nitems, st);
  return launch_hd<64>(mQ, mK, mV, mKb, mVb, p, p.nitems, st);
}

int last_attn_grid() { return g_last_grid; }

cudaError_t read_cta_times(cudaStream_t st, unsigned long long* host, int n) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  if (n > kMaxCtaTimes) n = kMaxCtaTimes;
  return cudaMemcpyFromSymbol(host, g_cta_times, (size_t)n * 4 * sizeof(unsigned long long));
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
