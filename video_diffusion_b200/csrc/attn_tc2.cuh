// attn_tc2.cuh -- two query-block streams per CTA (included by attn_tc.cu,
// inside its anonymous namespace; shares its helpers and status word).
//
// Same Sol-Attn loop as attn_tc_kernel (Sol-Attn visual explainer, "One
// online-softmax state"; Eqs. 9, 10, 11): per query block, the pooled-key
// chunks holding an unselected block first, then the selected key blocks, all
// folded into one online softmax.  What changes is how the tensor pipe is
// kept busy.  A softmax pass over a 128 x 128 tile takes about as long as the
// tensor work of the tile (QK^T and PV, 1024 cycles at d = 128), and the next
// tile's S of the same query block can only be computed after that pass.  So
// each CTA runs two independent query blocks ("streams") at once, each with
// its own warpgroup of softmax warps and its own S and O in TMEM: while one
// stream's softmax works on its tile, the tensor cores run the other stream's
// PV and next S.  The two softmax warps sharing a scheduler then work in
// alternation instead of in lock step, and each thread owns a whole 128-key
// row of its stream's tile, so there is one running max, one row sum and one
// O accumulator per row (no partial states to merge).
//
// Persistent CTAs, one per SM, 384 threads in three warpgroups:
//   WG0  warp 0  TMA producer: fetches work items, hands each to a stream,
//                loads its Q tile and, in the order the MMA warp consumes
//                them, each tile's K and V (or K-bar and V-bar) tiles into a
//                ring of single-tile slots (K slots free after S, V slots
//                after PV)
//        warp 1  TMEM owner and tcgen05.mma issuer (one elected lane); the
//                two streams' MMAs are issued in a fixed alternation
//        warp 2  in-kernel routing only: scores each item ahead of the producer
//        warp 3  idle
//   WG1, WG2    softmax and epilogue of streams 0 and 1, one query row per
//               thread (the warp's TMEM lane quadrant), 128 key columns
// Registers are rebalanced at start: the control warpgroup gives up most of
// its registers (setmaxnreg) to the two softmax warpgroups, which hold a
// 128-column score row per thread.
// TMEM columns: S_s at 128 s (P_s written over its first 64 columns as bf16
// pairs), O_s at 256 + 128 s.  Within a stream, S(n) is issued after PV(n-1)
// by the same thread, so when S(n) is complete O_s already holds every PV up
// to n - 1: the softmax may rescale O_s without a further wait.
// Every mbarrier wait is bounded, as in attn_tc_kernel.

namespace tc2 {

constexpr int NTHREADS = 384;
constexpr int DD = 6;                             // tile descriptors in flight per stream
constexpr int REG_CONTROL = 88, REG_SOFTMAX = 208;  // 128 x 88 + 256 x 208 = 384 x 168
static_assert(128 * REG_CONTROL + 256 * REG_SOFTMAX <= NTHREADS * 168, "register split");
constexpr uint32_t BAR_AREA2 = 3072;

template <int HD>
struct Cfg2 {
  static_assert(HD == 64 || HD == 128, "head dimension");
  static constexpr int NSLAB = HD / 64;
  static constexpr uint32_t TILE_BYTES = NSLAB * SLAB;
  static constexpr int NSLOT = HD == 128 ? 5 : 12;        // ring slots of one K or V tile
  static constexpr uint32_t OFF_Q = 0;                    // stream s: Q tile at s * TILE_BYTES
  static constexpr uint32_t OFF_RING = 2 * TILE_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_RING + NSLOT * TILE_BYTES;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + BAR_AREA2;
};
static_assert(Cfg2<128>::SMEM_BYTES <= 227 * 1024 && Cfg2<64>::SMEM_BYTES <= 227 * 1024, "shared memory");

struct StreamBars {
  uint64_t item_full[2], item_empty[2];  // producer -> MMA warp + the stream's softmax warps
  uint64_t q_full, q_empty;              // Q tile loaded / every S of its item issued and done
  uint64_t s_full, p_full;               // S in TMEM / P written over it by all 4 softmax warps
  uint64_t o_full, o_free;               // the item's last PV done / O read by the epilogue
  uint64_t desc_full[DD], desc_empty[DD];
  int item_slot[2], item_T[2];
  TileDesc desc[DD];
};

template <int NSLOT>
struct Bars2 {
  StreamBars st[2];
  uint64_t slot_full[NSLOT], slot_empty[NSLOT];
  uint64_t rq_full[2], rq_empty[2];  // in-kernel routing: router warp -> producer
  int rq_item[2], rq_T[2];
  uint32_t rq_bits[2][64];
  uint64_t teardown;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars2<12>) <= BAR_AREA2 && sizeof(Bars2<5>) <= BAR_AREA2, "barrier area");

__device__ __forceinline__ uint32_t low_bits(int n) { return n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u)); }

template <int R>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R)); }
template <int R>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R)); }

// Producer-side state of one stream.
struct ProdStream {
  TileIter ti;
  int T, nk, nv, active, done, q_uses, item_seq, bh, qi;
  int pkind, pidx, pidx2;  // the tile whose K was loaded last (its V is loaded next)
  uint32_t gdesc;          // descriptors written
  __device__ void init() {
    T = nk = nv = active = done = q_uses = item_seq = bh = qi = 0;
    pkind = pidx = 0;
    pidx2 = -1;
    gdesc = 0;
  }
};

// MMA-side state of one stream.
struct MmaStream {
  int T, ns, npv, active, done, item_seq, items_done, q_uses;
  uint32_t gp;  // PVs issued (P handoffs consumed)
  __device__ void init() { T = ns = npv = active = done = item_seq = items_done = q_uses = 0; gp = 0; }
};

template <int HD>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                    const __grid_constant__ CUtensorMap tmVb, const Params p) {
  using C = Cfg2<HD>;
  constexpr int NSLOT = C::NSLOT;
  constexpr int NSLAB = C::NSLAB;
  constexpr uint32_t TILE_BYTES = C::TILE_BYTES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(&g_sol_status, 0, 0x2000);
    return;
  }
  uint8_t* smem = smem_raw;
  Bars2<NSLOT>& bars = *reinterpret_cast<Bars2<NSLOT>*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      StreamBars& sb = bars.st[s];
      for (int k = 0; k < 2; ++k) {
        mbar_init(&sb.item_full[k], 1);
        mbar_init(&sb.item_empty[k], 1 + 4);
      }
      mbar_init(&sb.q_full, 1);
      mbar_init(&sb.q_empty, 1);
      mbar_init(&sb.s_full, 1);
      mbar_init(&sb.p_full, 4);
      mbar_init(&sb.o_full, 1);
      mbar_init(&sb.o_free, 4);
      for (int k = 0; k < DD; ++k) {
        mbar_init(&sb.desc_full[k], 1);
        mbar_init(&sb.desc_empty[k], 4);
      }
    }
    for (int k = 0; k < NSLOT; ++k) {
      mbar_init(&bars.slot_full[k], 1);
      mbar_init(&bars.slot_empty[k], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bars.rq_full[k], 1);
      mbar_init(&bars.rq_empty[k], 1);
    }
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
  const unsigned long long t_start = globaltimer_ns();
  int n_items_done = 0, n_tiles_done = 0;  // producer's count, for the per-CTA record

  if (wg == 0) {
    setmaxnreg_dec<REG_CONTROL>();
    if (warp == 0) {
      // ============================================================== producer (whole warp, one lane issues)
      const bool leader = elect_one();
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t slot_i = 0;  // ring loads issued
      int rq_it = 0;        // items taken from the router warp
      bool router_done = false;
      bool ok = true;
      ProdStream ps0, ps1;
      ps0.init();
      ps1.init();

      // next work item and its tile count (and, with in-kernel routing, its
      // selection words: lane l holds word l in rb0 and word 32 + l in rb1)
      auto fetch = [&](int& item, int& T, uint32_t& rb0, uint32_t& rb1) -> bool {
        rb0 = rb1 = 0u;
        if (p.route_inkernel) {
          if (router_done) {
            item = -1;
            T = 0;
            return true;
          }
          const int k = rq_it & 1;
          if (!(ok = wait_warp(&bars.rq_full[k], (rq_it >> 1) & 1, bars, lim, 4))) return false;
          item = bars.rq_item[k];
          T = bars.rq_T[k];
          if (lane < p.W) rb0 = bars.rq_bits[k][lane];
          if (32 + lane < p.W) rb1 = bars.rq_bits[k][32 + lane];
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.rq_empty[k]);
          ++rq_it;
          if (item < 0) router_done = true;
        } else {
          int idx = 0;
          if (lane == 0) idx = atomicAdd(p.work_counter, 1);
          idx = __shfl_sync(0xffffffffu, idx, 0);
          item = idx < p.nitems ? p.order[idx] : -1;
          T = item >= 0 ? p.tiles[item] : 0;
        }
        return true;
      };
      // the next ring slot <- one K or V tile: key block j1 (and j2 in the
      // second 64 rows of a 64-token pair tile) or pooled chunk j1
      auto load_slot = [&](int bh, int kind, int j1, int j2, bool is_v) -> bool {
        const int sl = slot_i % NSLOT;
        const uint32_t u = slot_i / NSLOT;
        if (u > 0 && !(ok = wait_warp(&bars.slot_empty[sl], (u - 1) & 1, bars, lim, 3))) return false;
        if (leader) {
          uint8_t* dst = smem + C::OFF_RING + sl * TILE_BYTES;
          mbar_arrive_expect_tx(&bars.slot_full[sl], TILE_BYTES);
          if (kind == 1 && p.pair) {
            const CUtensorMap* m = is_v ? &tmV : &tmK;
            const int jb = j2 >= 0 ? j2 : j1;  // a tile with one block repeats it (masked out)
#pragma unroll
            for (int hd = 0; hd < NSLAB; ++hd) {
              tma_load_3d(dst + hd * SLAB, m, &bars.slot_full[sl], hd * 64, j1 * 64, bh, pol_kv);
              tma_load_3d(dst + hd * SLAB + 64 * 128, m, &bars.slot_full[sl], hd * 64, jb * 64, bh, pol_kv);
            }
          } else {
            const CUtensorMap* m = kind ? (is_v ? &tmV : &tmK) : (is_v ? &tmVb : &tmKb);
#pragma unroll
            for (int hd = 0; hd < NSLAB; ++hd)
              tma_load_3d(dst + hd * SLAB, m, &bars.slot_full[sl], hd * 64, j1 * BN, bh, pol_kv);
          }
        }
        ++slot_i;
        return true;
      };
      // K of the stream's next tile, after publishing the tile's descriptor
      auto load_k = [&](ProdStream& ps, StreamBars& sb) -> bool {
        int kind = 0, idx = 0, idx2 = -1;
        const bool has = ps.ti.next(kind, idx, idx2);
        SOL_DCHECK(has, 2);
        SOL_DCHECK(kind == 1 ? (idx >= 0 && idx < p.Nk && idx2 < p.Nk && (p.pair || idx2 < 0))
                             : (idx >= 0 && idx < p.chunks),
                   3);
        (void)has;
        uint32_t vm[4] = {0u, 0u, 0u, 0u};
        if (kind == 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) vm[q] = ps.ti.unselected(idx * 4 + q);
        }
        const uint32_t g = ps.gdesc;
        const int dk = g % DD;
        if (g >= DD && !(ok = wait_warp(&sb.desc_empty[dk], ((g / DD) - 1) & 1, bars, lim, 6))) return false;
        if (leader) {
          TileDesc& td = sb.desc[dk];
          td.kind = kind;
          td.idx = idx;
          td.idx2 = idx2;
#pragma unroll
          for (int q = 0; q < 4; ++q) td.vm[q] = vm[q];
          mbar_arrive(&sb.desc_full[dk]);  // release: the fields above are visible to its waiters
        }
        ++ps.gdesc;
        if (!load_slot(ps.bh, kind, idx, idx2, false)) return false;
        ps.pkind = kind;
        ps.pidx = idx;
        ps.pidx2 = idx2;
        ++ps.nk;
        return true;
      };
      // one step of stream s, mirroring the MMA warp's step (same slot order)
      auto step = [&](ProdStream& ps, StreamBars& sb) -> bool {
        if (!ps.active) {
          if (ps.done) return true;
          for (;;) {
            int item = -1, T = 0;
            uint32_t rb0, rb1;
            if (!fetch(item, T, rb0, rb1)) return false;
            const int k = ps.item_seq & 1;
            if (ps.item_seq >= 2 && !(ok = wait_warp(&sb.item_empty[k], ((ps.item_seq >> 1) - 1) & 1, bars, lim, 1)))
              return false;
            if (lane == 0) {
              sb.item_slot[k] = item;
              sb.item_T[k] = T;
              mbar_arrive(&sb.item_full[k]);
            }
            ++ps.item_seq;
            if (item < 0) {
              ps.done = 1;
              return true;
            }
            SOL_DCHECK(item < p.nitems && T >= 0, 1);
            ++n_items_done;
            n_tiles_done += T;
            if (T == 0) continue;
            ps.bh = item / p.Nq;
            ps.qi = item % p.Nq;
            ps.T = T;
            ps.nk = ps.nv = 0;
            ps.active = 1;
            if (p.route_inkernel) {
              ps.ti.init(nullptr, p.W, p.Nk, p.chunks, p.pair);
              ps.ti.rb0 = rb0;
              ps.ti.rb1 = rb1;
            } else if (p.W <= 64) {
              // the item's whole selection row in two registers per lane
              // (one coalesced load), so that walking its tiles costs
              // shuffles rather than a dependent L2 round trip per word
              const uint32_t* mrow = p.mask + (size_t)item * p.W;
              ps.ti.init(nullptr, p.W, p.Nk, p.chunks, p.pair);
              ps.ti.rb0 = lane < p.W ? __ldg(mrow + lane) : 0u;
              ps.ti.rb1 = 32 + lane < p.W ? __ldg(mrow + 32 + lane) : 0u;
            } else {
              ps.ti.init(p.mask + (size_t)item * p.W, p.W, p.Nk, p.chunks, p.pair);
            }
            // the stream's Q tile, once every S of its previous item is done
            if (ps.q_uses > 0 && !(ok = wait_warp(&sb.q_empty, (ps.q_uses - 1) & 1, bars, lim, 2))) return false;
            if (leader) {
              mbar_arrive_expect_tx(&sb.q_full, TILE_BYTES);
              uint8_t* qdst = smem + C::OFF_Q + (&sb == &bars.st[0] ? 0 : TILE_BYTES);
#pragma unroll
              for (int hd = 0; hd < NSLAB; ++hd)
                tma_load_3d(qdst + hd * SLAB, &tmQ, &sb.q_full, hd * 64, ps.qi * BM, ps.bh, pol_q);
            }
            ++ps.q_uses;
            return load_k(ps, sb);
          }
        }
        // V of the tile whose S is in flight, then K of the next tile
        if (!load_slot(ps.bh, ps.pkind, ps.pidx, ps.pidx2, true)) return false;
        ++ps.nv;
        if (ps.nk < ps.T && !load_k(ps, sb)) return false;
        if (ps.nv == ps.T) ps.active = 0;
        return true;
      };
      while (!(ps0.done && ps1.done)) {
        if (!step(ps0, bars.st[0])) break;
        if (!step(ps1, bars.st[1])) break;
      }
      if (!ok || bars.abort_flag) {
        // let every copy this warp started land before the CTA exits
        for (int back = 1; back <= NSLOT && back <= (int)slot_i; ++back) {
          const uint32_t gk = slot_i - back;
          mbar_wait(&bars.slot_full[gk % NSLOT], (gk / NSLOT) & 1, nullptr, &g_sol_status, 0, lim);
        }
        if (ps0.q_uses > 0) mbar_wait(&bars.st[0].q_full, (ps0.q_uses - 1) & 1, nullptr, &g_sol_status, 0, lim);
        if (ps1.q_uses > 0) mbar_wait(&bars.st[1].q_full, (ps1.q_uses - 1) & 1, nullptr, &g_sol_status, 0, lim);
      }
      __syncwarp();
    } else if (warp == 1) {
      // ============================================================== MMA issuer (whole warp, one lane issues)
      const bool leader = elect_one();
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, HD, false, true);
      constexpr uint32_t TILE16 = TILE_BYTES >> 4;
      // descriptors of ring slot 0 (K: K-major B of S = Q K^T; V: MN-major B
      // of O += P V) and of the two Q tiles; a slot or a K-step only moves the
      // 14-bit start-address field (shared memory < 256 KB: no carry)
      const uint64_t dK0 = smem_desc_sw128(smem_u32(smem + C::OFF_RING), 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_u32(smem + C::OFF_RING), SLAB, 1024);
      const uint64_t dQ0 = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
      uint32_t cslot = 0;  // ring slots consumed
      bool issued = false, ok = true, stalled = false;
      MmaStream ms0, ms1;
      ms0.init();
      ms1.init();
      auto issue_s = [&](MmaStream& ms, StreamBars& sb, int s) -> bool {
        const int sl = cslot % NSLOT;
        if (!(ok = wait_warp(&bars.slot_full[sl], (cslot / NSLOT) & 1, bars, lim, 15))) return false;
        tc_fence_after();
        // operands computed by the whole warp (warp-uniform values), issued by one lane
        const uint64_t dK = dK0 + (uint64_t)(sl * TILE16);
        const uint64_t dQ = dQ0 + (uint64_t)(s * TILE16);
        const uint32_t tS = tmem + TM_S + s * 128;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * SLAB + (kk & 3) * 32) >> 4;
            mma_ss(tS, dQ + off, dK + off, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars.slot_empty[sl]);
          if (!(p.test_stall && !stalled)) tc_commit(&sb.s_full);
          if (ms.ns == ms.T - 1) tc_commit(&sb.q_empty);  // every S of this item issued
        }
        stalled = true;
        __syncwarp();
        issued = true;
        ++cslot;
        ++ms.ns;
        return true;
      };
      auto step = [&](MmaStream& ms, StreamBars& sb, int s) -> bool {
        if (!ms.active) {
          if (ms.done) return true;
          for (;;) {
            const int k = ms.item_seq & 1;
            if (!(ok = wait_warp(&sb.item_full[k], (ms.item_seq >> 1) & 1, bars, lim, 10))) return false;
            const int item = sb.item_slot[k];
            const int T = sb.item_T[k];
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.item_empty[k]);
            ++ms.item_seq;
            if (item < 0) {
              ms.done = 1;
              return true;
            }
            if (T == 0) continue;
            ms.T = T;
            ms.ns = ms.npv = 0;
            ms.active = 1;
            if (!(ok = wait_warp(&sb.q_full, ms.q_uses & 1, bars, lim, 11))) return false;
            ++ms.q_uses;
            return issue_s(ms, sb, s);
          }
        }
        // O_s += P_s V of the tile the stream's softmax has just handed over
        if (!(ok = wait_warp(&sb.p_full, ms.gp & 1, bars, lim, 12))) return false;
        if (ms.npv == 0 && ms.items_done > 0 && !(ok = wait_warp(&sb.o_free, (ms.items_done - 1) & 1, bars, lim, 14)))
          return false;
        const int sl = cslot % NSLOT;
        if (!(ok = wait_warp(&bars.slot_full[sl], (cslot / NSLOT) & 1, bars, lim, 13))) return false;
        tc_fence_after();
        const uint64_t dV = dV0 + (uint64_t)(sl * TILE16);
        const uint32_t tP = tmem + TM_S + s * 128;
        const uint32_t tO = tmem + TM_O + s * 128;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tO, tP + kk * 8, dV + ((kk * 2048) >> 4), IDESC_PV, (ms.npv == 0 && kk == 0) ? 0u : 1u);
          tc_commit(&bars.slot_empty[sl]);
        }
        __syncwarp();
        ++cslot;
        ++ms.gp;
        ++ms.npv;
        if (ms.ns < ms.T && !issue_s(ms, sb, s)) return false;
        if (ms.npv == ms.T) {
          if (leader) tc_commit(&sb.o_full);
          __syncwarp();
          ms.active = 0;
          ++ms.items_done;
        }
        return true;
      };
      while (!(ms0.done && ms1.done)) {
        if (!step(ms0, bars.st[0], 0)) break;
        if (!step(ms1, bars.st[1], 1)) break;
      }
      (void)ok;
      if (issued) {
        // all MMAs of this CTA complete before TMEM is released
        if (leader) tc_commit(&bars.teardown);
        __syncwarp();
        mbar_wait(&bars.teardown, 0, nullptr, &g_sol_status, 0, lim);
      }
      __syncwarp();
    } else if (warp == 2) {
      // ============================================================== router (in-kernel routing only)
      bool ok = true;
      for (int it = 0; p.route_inkernel; ++it) {
        const int slot = it & 1;
        if (it >= 2 && !(ok = wait_warp(&bars.rq_empty[slot], ((it >> 1) - 1) & 1, bars, lim, 5))) break;
        int idx = 0;
        if (lane == 0) idx = atomicAdd(p.work_counter, 1);
        idx = __shfl_sync(0xffffffffu, idx, 0);
        const int item = idx < p.nitems ? p.order[idx] : -1;
        int T = 0;
        if (item >= 0) {
          uint32_t rb0, rb1;
          T = route_row<HD>(p, item, lane, rb0, rb1);
          if (lane < p.W) bars.rq_bits[slot][lane] = rb0;
          if (32 + lane < p.W) bars.rq_bits[slot][32 + lane] = rb1;
        }
        __syncwarp();
        if (lane == 0) {
          bars.rq_item[slot] = item;
          bars.rq_T[slot] = T;
          mbar_arrive(&bars.rq_full[slot]);
        }
        if (item < 0) break;
      }
      (void)ok;
    }
  } else {
    // ================================================================ softmax + epilogue of stream wg - 1
    setmaxnreg_inc<REG_SOFTMAX>();
    const int s = wg - 1;
    StreamBars& sb = bars.st[s];
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;   // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + TM_S + s * 128;
    const uint32_t tO = tmem + lane_off + TM_O + s * 128;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;  // tiles of this stream so far
    int item_seq = 0, items_done = 0;
    bool ok = true;
    for (;;) {
      const int k = item_seq & 1;
      if (!(ok = wait_warp(&sb.item_full[k], (item_seq >> 1) & 1, bars, lim, 20))) break;
      const int item = sb.item_slot[k];
      const int T = sb.item_T[k];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sb.item_empty[k]);
      ++item_seq;
      if (item < 0) break;
      const int bh = item / p.Nq, qi = item % p.Nq;
      const int n_rows = min(BM, p.L - qi * BM);
      __nv_bfloat16* orow = p.out + ((size_t)bh * p.L + (size_t)qi * BM + row) * HD;
      if (T == 0) {
        if (row < n_rows)
          for (int c = 0; c < HD; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0, 0, 0, 0);
        continue;
      }
      float m_used = -INFINITY, l = 0.f;
      for (int n = 0; n < T; ++n, ++g) {
        if (!(ok = wait_warp(&sb.s_full, g & 1, bars, lim, 21))) break;
        const int dk = g % DD;
        if (!(ok = wait_warp(&sb.desc_full[dk], (g / DD) & 1, bars, lim, 22))) break;
        const int kind = sb.desc[dk].kind, tidx = sb.desc[dk].idx, tidx2 = sb.desc[dk].idx2;
        uint32_t vm[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) vm[q] = sb.desc[dk].vm[q];
        SOL_DCHECK((kind == 0 && tidx < p.nchunk) || (kind == 1 && tidx < p.Nk && tidx2 < p.Nk), 4);
        tc_fence_after();
        float x[2][64];
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld32(tS + 64, r2);
          tmem_ld32(tS + 96, r3);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            x[0][c] = __uint_as_float(r0[c]);
            x[0][32 + c] = __uint_as_float(r1[c]);
            x[1][c] = __uint_as_float(r2[c]);
            x[1][32 + c] = __uint_as_float(r3[c]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sb.desc_empty[dk]);  // descriptor read; S read into registers
        // valid key columns: all 128 except in the last (partial) key block
        // and in a 64-token pair tile with one block; pooled chunks carry
        // their unselected, in-range columns in vm
        bool full = false;
        float bias = 0.f;
        int sc = -1;
        float sc_delta = 0.f;
        if (kind == 1) {
          if (p.pair) {
            const int nv0 = tidx == p.Nk - 1 ? p.nk_last : 64;
            const int nv1 = tidx2 < 0 ? 0 : (tidx2 == p.Nk - 1 ? p.nk_last : 64);
            vm[0] = low_bits(nv0);
            vm[1] = low_bits(nv0 - 32);
            vm[2] = low_bits(nv1);
            vm[3] = low_bits(nv1 - 32);
            full = nv0 == 64 && nv1 == 64;
          } else {
            const int nb = tidx == p.Nk - 1 ? p.nk_last : BN;
#pragma unroll
            for (int q = 0; q < 4; ++q) vm[q] = low_bits(nb - 32 * q);
            full = nb == BN;
          }
        } else {
          bias = p.bias_full;
          const int jl = p.Nk - 1 - tidx * BN;
          if (jl >= 0 && jl < BN && p.bias_last != p.bias_full) {
            sc = jl;
            sc_delta = p.bias_last - p.bias_full;
          }
        }
        // full exact tile: x stays the raw score (scale folded into exp2);
        // otherwise x becomes the log2-domain logit with bias and mask applied
        float lmax;
        if (full) {
          lmax = fmaxf(tree_max64(x[0]), tree_max64(x[1])) * sl2;  // scaling by sl2 > 0 commutes with max
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int col = 64 * h + c;
              float u = fmaf(x[h][c], sl2, bias);
              if (col == sc) u += sc_delta;
              x[h][c] = ((vm[col >> 5] >> (col & 31)) & 1u) ? u : -INFINITY;
            }
          }
          lmax = fmaxf(tree_max64(x[0]), tree_max64(x[1]));
        }
        const float m_new = fmaxf(m_used, lmax);
        const bool need = m_new > m_used + RESCALE_THRESHOLD;
        float alpha = 1.f;
        if (need) {
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
          l *= alpha;
        }
        if (n > 0 && __any_sync(0xffffffffu, need)) {
          // S of this tile was issued after PV of the previous one, so O_s
          // already holds every earlier PV
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
        const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
        const float2 sl2v = make_float2(full ? sl2 : 1.f, full ? sl2 : 1.f);
        const float2 negv = make_float2(neg_m, neg_m);
        {
          uint32_t pk[32];
          l += exp_pack64<NPOLY>(x[0], sl2v, negv, pk);
          tmem_st32(tS, pk);  // P over the first 64 columns of S_s, as bf16 pairs
        }
        {
          uint32_t pk[32];
          l += exp_pack64<NPOLY>(x[1], sl2v, negv, pk);
          tmem_st32(tS + 32, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sb.p_full);
      }
      if (!ok) break;
      // epilogue: out = O / l for this thread's row
      if (!(ok = wait_warp(&sb.o_full, items_done & 1, bars, lim, 24))) break;
      tc_fence_after();
      uint32_t o[HD / 32][32];
#pragma unroll
      for (int q = 0; q < HD / 32; ++q) tmem_ld32(tO + q * 32, o[q]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sb.o_free);
      const float inv = 1.0f / l;
      SOL_DCHECK(inv > 0.f && inv < INFINITY, 6);
      if (row < n_rows) {
#pragma unroll
        for (int q = 0; q < HD / 32; ++q) {
#pragma unroll
          for (int c = 0; c < 32; c += 16) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w[e] = pack_bf16x2(__uint_as_float(o[q][c + 2 * e]) * inv, __uint_as_float(o[q][c + 2 * e + 1]) * inv);
            if (p.out_align32) {
              st_global_v8(orow + q * 32 + c, w);
            } else {
              *reinterpret_cast<uint4*>(orow + q * 32 + c) = make_uint4(w[0], w[1], w[2], w[3]);
              *reinterpret_cast<uint4*>(orow + q * 32 + c + 8) = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
        }
      }
      ++items_done;
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

}  // namespace tc2
