// Tensor-core (tcgen05) causal attention, two query tiles per work item, on a
// persistent grid.
//
// Sources: Kimi-K2 "Query content heads" page, "Join query parts", and the
// Kimi-K2 "RoPE coefficients" page, "Key heads" (mla-prefill excerpt): each
// head's query and key join their non-rotary and rotary parts (the key's
// rotary part is the one rotary key shared by all heads), the scores are
// scaled, causally masked, normalized with a softmax in fp32 and mix the
// values. The arithmetic is the one of attention_kernel except for the types
// of the score product's operands (below); this kernel changes how it is
// scheduled on the SM.
//
// Work item = one head x one 256-row block of queries, split into tile A
// (rows 0-127) and tile B (rows 128-255). Both tiles read the same key /
// value tiles (128 keys per step), so each K/V byte staged in shared memory
// feeds twice the tensor-core work. One CTA runs per SM and takes items from
// a device-wide counter, heaviest blocks first (the block list is sorted by
// causal work), so the grid balances itself. Warps (three warpgroups; the
// first runs on 56 registers per thread so that the softmax warpgroups can
// hold a whole row of scores in 216):
//   warp 0     producer: claims the next item two key steps before the
//              current item's end (the claim and the lookup of the item's
//              sequence, rows and step counts happen while key steps are in
//              flight, and the next item's Q rows are prefetched into L2
//              then), publishes each decoded item to the other warps through
//              a two-slot ring in shared memory, loads the tiles' Q and, per
//              key step, the key atoms and the two transposed value boxes into
//              a ring of 16 KB slots. The key/value stream runs on across
//              items, and the next item's Q is loaded as soon as the current
//              item's last score product on that tile has finished.
//   warp 1     MMA issuer (whole warp, one elected lane issues)
//   warps 2-3  idle
//   warps 4-7  softmax of tile A (one query row per thread, TMEM lane = row)
//   warps 8-11 softmax of tile B
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+V),
// O_B [384,384+V). P (fp16) is written back over the first 64 columns of its
// own S buffer and read from there by the P V product (A operand in TMEM).
// Per global key step g the MMA warp issues
//   PV_A(g)  S_A(g+1)  PV_B(g)  S_B(g+1)
// (each only when that tile uses the step; step g+1 may belong to the next
// item), so one tile's softmax runs while the tensor cores work on the other
// tile, and every key and value group is consumed in the order it was loaded.
// Tensor-core instructions from one thread run in issue order, so S_X(g+1)
// overwrites P_X(g) only after PV_X(g) has read it.
//
// Score operands: the non-rotary atoms multiply q as given (bf16) with k_nope
// stored in bf16; the rotary atom multiplies the query's rotary part, turned
// at its position once before this kernel (q_rope_warp, run by the
// up-projection GEMM's epilogue warps or a preparation kernel), with the
// rotated shared key, both fp16; all products accumulate in one fp32 TMEM
// tile. So Q needs no work on this SM: its first score product starts when
// its copy lands. At the end of an item a tile's softmax warps write the
// item's output from O; the next item's first P V product (which overwrites
// O) waits for that.
//
// Softmax reference: a row's reference m is its maximum over the first key
// tile; it is raised (and O and the row sum rescaled) only when a later tile's
// maximum exceeds it by more than kPrLazy (log2 units), so P <= 2^kPrLazy,
// well inside fp16. The weights are formed as e = 2^(s - m - kPrBias) (fp32,
// always normal), their row sum is kept in fp32 at that scale, and their fp16
// codes come from e * 2^-12 = P * 2^-112 by integer arithmetic
// (f16x2_from_scaled), which keeps the conversion off the MUFU pipe that the
// exponentials saturate. The codes equal round-to-nearest fp16 of P
// (subnormals included; exact ties round away from zero). The row sum adds the
// fp32 weights before their rounding to fp16 (relative difference <= 2^-12 of
// the result).
#pragma once
#include "tc_attention.cuh"

namespace mla {
namespace tc {

constexpr int kPrBKV = 128;                 // keys per step
constexpr int kPrThreads = 384;
// Registers per thread of the producer / MMA warpgroup and of the two softmax
// warpgroups: 128 x 56 + 256 x 216 = 62464, within the 384 x 168 = 64512 the
// launch holds (ptxas gives this kernel 168 per thread; checked at build).
constexpr int kPrRegsCtl = 56;
constexpr int kPrRegsSoftmax = 216;
static_assert(128 * kPrRegsCtl + 256 * kPrRegsSoftmax <= kPrThreads * 168, "register split exceeds the launch");
constexpr int kPrSlotBytes = 16384;
constexpr int kPrMaxSlots = 12;
constexpr float kPrLazy = 8.f;
constexpr int kPrGroupDepth = 4;
constexpr int kPrSched = 2;                 // item slots between the producer and the other warps
constexpr int kPrSchedReaders = 9;          // the MMA warp and the eight softmax warps
constexpr float kPrBias = 100.f;            // e = P * 2^-kPrBias stays a normal fp32 number
constexpr float kPrTwoM12 = 2.44140625e-4f;         // 2^-12
constexpr float kPrTwoMBias = 7.888609052210118e-31f;   // 2^-100
template <int kN, int kV>
struct PairCfg {
  static constexpr int D = kN + 64;
  static constexpr int kQAtoms = D / 64;
  static constexpr int kQTileBytes = kQAtoms * kTile * 128;          // 128 rows x D fp16
  static constexpr int kQBytes = 2 * kQTileBytes;
  static constexpr int kKAtoms = kN / 64;                              // k_nope atoms per step
  static constexpr int kVBoxBytes = kV * 128;                          // [V rows x 64 keys]
  static constexpr int kBoxes = kQAtoms + 2;                           // ring slots per step
  static constexpr int kSlotsFit = (232448 - 2048 - kQBytes) / kPrSlotBytes;
  static constexpr int kSlots = kSlotsFit < kPrMaxSlots ? kSlotsFit : kPrMaxSlots;
  static constexpr size_t kSmem = (size_t)kQBytes + (size_t)kSlots * kPrSlotBytes + 1024;
  static_assert(kBoxes <= kSlots, "one step of boxes must fit the ring");
  static_assert(kSlots <= 3 * kBoxes, "a slot must be reused within three steps");
  static_assert(kV <= 128, "two O accumulators must fit next to the S buffers");
  static constexpr uint32_t kOCol = 256;
};

// The ring's boxes travel in groups: per step one key group (the k_nope
// atoms and the rotary key atom) and one value group (two boxes). Each group
// has one "full" barrier (all its copies landed) and one "empty" barrier (the
// MMAs reading it are done), so the MMA warp waits once per group instead of
// once per box. The barriers rotate over kPrGroupDepth global steps: a box's
// slot was last used at most three steps earlier (static_assert above), and
// the release the producer waits for before re-arming a step's barrier is
// issued after the MMA warp's wait on that barrier four steps earlier.
struct PairBarriers {
  uint64_t q_full[2], q_free[2];
  uint64_t kfull[kPrGroupDepth], kempty[kPrGroupDepth], vfull[kPrGroupDepth], vempty[kPrGroupDepth];
  uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  uint64_t sched_full[kPrSched], sched_empty[kPrSched];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// One work item, decoded from its index: head h of the block whose first tile
// is order[item / H].
struct PairItem {
  int valid;                  // 0: past the last item (or the counter ran past the list)
  int h, q0, L, kv_pad0;
  int off;                    // key index of the sequence's first query (0 without cached rows)
  int nA, nB, n;              // key steps of tile A, tile B (0: all padding), the item
  int64_t seq0;
};

__device__ __forceinline__ PairItem pair_item(const AttParams& p, int item) {
  PairItem it;
  it.valid = 0;
  it.h = it.q0 = it.L = it.kv_pad0 = it.off = it.nA = it.nB = it.n = 0;
  it.seq0 = 0;
  if (item < 0) return it;
  const int rank = item / p.H;
  if (rank >= p.n_blocks) return it;
  const int tile = p.order[rank];
  if (tile < 0 || tile >= p.n_blocks) return it;   // n_blocks bounds the tile tables too
  const int seq = p.tile_seq[tile];
  if (seq < 0) return it;
  it.valid = 1;
  it.h = item - rank * p.H;
  it.q0 = p.tile_q0[tile];                                   // multiple of 256
  it.seq0 = p.cu[seq];
  it.L = (int)(p.cu[seq + 1] - it.seq0);
  it.kv_pad0 = p.seq_tile0[seq] * kTile;
  it.off = p.q_off ? p.q_off[seq] : 0;
  // query row r attends keys 0 .. off + r; a tile's key steps reach its last valid row's
  it.nA = (it.off + min(it.q0 + kTile - 1, it.L - 1)) / kPrBKV + 1;
  it.nB = (it.q0 + kTile < it.L) ? (it.off + min(it.q0 + 2 * kTile - 1, it.L - 1)) / kPrBKV + 1 : 0;
  it.n = it.nA > it.nB ? it.nA : it.nB;
  return it;
}

// The k-th work item of the CTA, as published (decoded) by the producer in
// the shared-memory ring `ring`: every reader warp reads every slot once, in
// order. Returns false on abort.
__device__ __forceinline__ bool pair_read_item(PairBarriers& bars, const PairItem* ring, int k, int lane,
                                               volatile int* abort_flag, PairItem& it) {
  const int s = k % kPrSched;
  if (!mbar_wait_warp(&bars.sched_full[s], (uint32_t)(k / kPrSched) & 1u, abort_flag)) return false;
  const volatile PairItem& r = ring[s];
  it.valid = r.valid; it.h = r.h; it.q0 = r.q0; it.L = r.L; it.kv_pad0 = r.kv_pad0; it.off = r.off;
  it.nA = r.nA; it.nB = r.nB; it.n = r.n; it.seq0 = r.seq0;
  __syncwarp();
  if (lane == 0) mbar_arrive(&bars.sched_empty[s]);
  return true;
}

template <int kN, int kV>
__global__ void __launch_bounds__(kPrThreads, 1)
attention_pair_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
                      const __grid_constant__ CUtensorMap map_kn, const __grid_constant__ CUtensorMap map_kr,
                      const __grid_constant__ CUtensorMap map_vt, AttParams p) {
  using C = PairCfg<kN, kV>;
  constexpr int S = C::kSlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ PairBarriers bars;
  __shared__ PairItem sched_ring[kPrSched];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_allow_next();
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::kQBytes;
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars.q_full[x], 1);
      mbar_init(&bars.q_free[x], 1);
      mbar_init(&bars.s_full[x], 1);
      mbar_init(&bars.p_full[x], 128);
      mbar_init(&bars.pv_done[x], 1);
      mbar_init(&bars.o_free[x], 128);
    }
    for (int b = 0; b < kPrGroupDepth; ++b) {
      mbar_init(&bars.kfull[b], 1); mbar_init(&bars.kempty[b], 1);
      mbar_init(&bars.vfull[b], 1); mbar_init(&bars.vempty[b], 1);
    }
    for (int s = 0; s < kPrSched; ++s) {
      mbar_init(&bars.sched_full[s], 1);
      mbar_init(&bars.sched_empty[s], kPrSchedReaders);
    }
    mbar_init(&bars.mma_done, 1);
    bars.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;


  if (warp < 4) {
    warpgroup_reg_dec<kPrRegsCtl>();
    if (warp == 0) {
      // ---------------- producer ----------------
      if (lane == 0) {
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_qr);
        tma_prefetch_desc(&map_kn);
        tma_prefetch_desc(&map_kr);
        tma_prefetch_desc(&map_vt);
        // box gb of the ring sits in slot gb % S; before it is filled, the group
        // that last used the slot (box gb - S) must have been released
        auto wait_released = [&](int gp) -> bool {
          const int jp = gp / C::kBoxes;
          uint64_t* bar = (gp % C::kBoxes) < C::kQAtoms ? &bars.kempty[jp & 3] : &bars.vempty[jp & 3];
          return mbar_wait(bar, (uint32_t)(jp >> 2) & 1u, abort_flag);
        };
        pdl_wait();   // k_nope, the values, k_rot and the schedule come from the previous kernels
        bool ok = true;
        int g = 0;                         // global key step
        int gk = -1, gv = -1;              // last key / value group issued
        int uq[2] = {0, 0};                // Q loads issued per tile
        // the first item of every CTA is its own index (the grid never exceeds
        // the item count); the counter hands out the rest
        PairItem next = pair_item(p, (int)blockIdx.x);
        for (int k = 0; ok; ++k) {
          const int s = k % kPrSched;
          if (!(ok = mbar_wait(&bars.sched_empty[s], ((uint32_t)(k / kPrSched) & 1u) ^ 1u, abort_flag))) break;
          const PairItem it = next;
          volatile PairItem& r = sched_ring[s];
          r.valid = it.valid; r.h = it.h; r.q0 = it.q0; r.L = it.L; r.kv_pad0 = it.kv_pad0; r.off = it.off;
          r.nA = it.nA; r.nB = it.nB; r.n = it.n; r.seq0 = it.seq0;
          mbar_arrive(&bars.sched_full[s]);
          if (!it.valid) break;
          bool claimed = false;              // the item after this one claimed yet
          auto load_q = [&](int x) -> bool {
            if (uq[x] > 0 && !mbar_wait(&bars.q_free[x], (uint32_t)(uq[x] - 1) & 1u, abort_flag)) return false;
            mbar_arrive_expect_tx(&bars.q_full[x], C::kQTileBytes);
            const int qrow0 = (int)(it.seq0 + it.q0 + x * kTile);
            for (int a = 0; a < C::kKAtoms; ++a)
              tma_load_3d(sQ + x * C::kQTileBytes + a * kTile * 128, &map_q, &bars.q_full[x], a * 64, it.h, qrow0);
            tma_load_3d(sQ + x * C::kQTileBytes + C::kKAtoms * kTile * 128, &map_qr, &bars.q_full[x], 0, it.h, qrow0);
            ++uq[x];
            return true;
          };
          if (!(ok = load_q(0))) break;
          for (int j = 0; j < it.n && ok; ++j, ++g) {
            const int kv_row = it.kv_pad0 + j * kPrBKV;
            const int g0 = g * C::kBoxes;
            for (int i = 0; i < C::kQAtoms && ok; ++i)
              if (g0 + i >= S) ok = wait_released(g0 + i - S);
            if (!ok) break;
            uint64_t* kb = &bars.kfull[g & 3];
            mbar_arrive_expect_tx(kb, C::kQAtoms * kPrBKV * 128);
            for (int i = 0; i < C::kKAtoms; ++i)
              tma_load_2d(sRing + ((g0 + i) % S) * kPrSlotBytes, &map_kn, kb, i * 64, it.h * p.Tpad + kv_row);
            tma_load_2d(sRing + ((g0 + C::kKAtoms) % S) * kPrSlotBytes, &map_kr, kb, 0, kv_row);
            gk = g;
            for (int v = 0; v < 2 && ok; ++v)
              if (g0 + C::kQAtoms + v >= S) ok = wait_released(g0 + C::kQAtoms + v - S);
            if (!ok) break;
            uint64_t* vb = &bars.vfull[g & 3];
            mbar_arrive_expect_tx(vb, 2 * C::kVBoxBytes);
            for (int v = 0; v < 2; ++v)
              tma_load_2d(sRing + ((g0 + C::kQAtoms + v) % S) * kPrSlotBytes, &map_vt, vb, kv_row + v * 64,
                          it.h * kV);
            gv = g;
            // tile B's Q after the first step's keys and values, so that a
            // wait for the previous item's last tile-B scores never holds up
            // the keys tile A needs first
            if (j == 0 && it.nB > 0 && !(ok = load_q(1))) break;
            if (!claimed && j == max(it.n - 2, 0)) {
              // two steps before the item's end (the ring is full, so the
              // lookups' latency costs nothing): claim and decode the next
              // item, and start its Q rows on their way to L2. Claiming this
              // late keeps the heaviest-first order of the claims close to the
              // order in which the CTAs run out of work.
              claimed = true;
              next = pair_item(p, (int)gridDim.x + atomicAdd(p.item_counter, 1));
              if (next.valid)
                for (int x = 0; x < (next.nB > 0 ? 2 : 1); ++x) {
                  const int r0 = (int)(next.seq0 + next.q0 + x * kTile);
                  for (int a = 0; a < C::kKAtoms; ++a) tma_prefetch_l2_3d(&map_q, a * 64, next.h, r0);
                  tma_prefetch_l2_3d(&map_qr, 0, next.h, r0);
                }
            }
          }
          if (ok && !claimed) next = pair_item(p, (int)gridDim.x + atomicAdd(p.item_counter, 1));
        }
        if (!ok) {   // let every copy already issued land before the CTA exits
          for (int x = 0; x < 2; ++x)
            if (uq[x] > 0) mbar_wait_drain(&bars.q_full[x], (uint32_t)(uq[x] - 1) & 1u);
          for (int jj = (gk > 3 ? gk - 3 : 0); jj <= gk; ++jj)
            mbar_wait_drain(&bars.kfull[jj & 3], (uint32_t)(jj >> 2) & 1u);
          for (int jj = (gv > 3 ? gv - 3 : 0); jj <= gv; ++jj)
            mbar_wait_drain(&bars.vfull[jj & 3], (uint32_t)(jj >> 2) & 1u);
        }
      }
    } else if (warp == 1) {
      // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
      const uint32_t idesc_s_nope = idesc_bf16_f32(kTile, kPrBKV);   // q as given, k_nope in bf16
      const uint32_t idesc_s_rope = idesc_f16_f32(kTile, kPrBKV);    // rotated q and key in fp16
      const uint32_t idesc_o = idesc_f16_f32(kTile, kV);
      const uint32_t ring0 = smem_u32(sRing), q0addr = smem_u32(sQ);
      auto slot_addr = [&](int gb) -> uint32_t { return ring0 + (uint32_t)(gb % S) * kPrSlotBytes; };
      int k_seen = -1, v_seen = -1;       // last global step whose key / value group was waited for
      int uq[2] = {0, 0};                 // Q uses per tile (q_full phases)
      int uo[2] = {0, 0};                 // items per tile whose P V has started (o_free phases)
      int ts[2] = {0, 0};                 // tile-steps per tile (p_full phases)
      // S_x(step g) = Q_x K_g^T over all D columns
      auto issue_s = [&](int x, int g) -> bool {
        if (k_seen < g) {
          if (!mbar_wait_warp(&bars.kfull[g & 3], (uint32_t)(g >> 2) & 1u, abort_flag)) return false;
          k_seen = g;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(x * kPrBKV);
  #pragma unroll 1
        for (int a = 0; a < C::kQAtoms; ++a) {
          const uint64_t qd = desc_kmajor_sw128(q0addr + (uint32_t)(x * C::kQTileBytes + a * kTile * 128));
          const uint64_t kd = desc_kmajor_sw128(slot_addr(g * C::kBoxes + a));
          const uint32_t idesc_s = a < C::kKAtoms ? idesc_s_nope : idesc_s_rope;
  #pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss_elect(d, desc_advance(qd, k * 32), desc_advance(kd, k * 32), idesc_s, (a | k) != 0);
        }
        mma_commit_elect(&bars.s_full[x]);
        return true;
      };
      // first S of tile x in a new item: its Q must have landed
      auto issue_s_first = [&](int x, int g, int nx) -> bool {
        if (!mbar_wait_warp(&bars.q_full[x], (uint32_t)uq[x] & 1u, abort_flag)) return false;
        ++uq[x];
        if (!issue_s(x, g)) return false;
        if (nx == 1) mma_commit_elect(&bars.q_free[x]);
        return true;
      };
      // O_x (+)= P_x(step g) V_g, P_x read from TMEM; `first`: the item's first step
      auto issue_pv = [&](int x, int g, bool first) -> bool {
        if (v_seen < g) {
          if (!mbar_wait_warp(&bars.vfull[g & 3], (uint32_t)(g >> 2) & 1u, abort_flag)) return false;
          v_seen = g;
        }
        if (first) {
          if (uo[x] > 0 && !mbar_wait_warp(&bars.o_free[x], (uint32_t)(uo[x] - 1) & 1u, abort_flag)) return false;
          ++uo[x];
        }
        if (!mbar_wait_warp(&bars.p_full[x], (uint32_t)ts[x] & 1u, abort_flag)) return false;
        ++ts[x];
        tc_fence_after();
        const uint32_t pa = tmem + (uint32_t)(x * kPrBKV);
        const uint32_t o = tmem + C::kOCol + (uint32_t)(x * 128);
  #pragma unroll 1
        for (int v = 0; v < 2; ++v) {
          const uint64_t vd = desc_kmajor_sw128(slot_addr(g * C::kBoxes + C::kQAtoms + v));
  #pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts_elect(o, pa + (uint32_t)((v * 4 + k) * 8), desc_advance(vd, k * 32), idesc_o,
                         (!first || (v | k) != 0) ? 1u : 0u);
        }
        mma_commit_elect(&bars.pv_done[x]);
        return true;
      };

      // the MMA warp needs only the step counts of an item
      struct Steps { int valid, nA, nB, n; };
      auto read_steps = [&](int k, Steps& st) -> bool {
        PairItem it;
        if (!pair_read_item(bars, sched_ring, k, lane, abort_flag, it)) return false;
        st.valid = it.valid; st.nA = it.nA; st.nB = it.nB; st.n = it.n;
        return true;
      };
      int kread = 0;
      Steps cur;
      bool ok = read_steps(kread++, cur);
      int g = 0;                          // global step of cur's first key step
      if (ok && cur.valid) {
        ok = issue_s_first(0, 0, cur.nA);
        if (ok && cur.nB > 0) ok = issue_s_first(1, 0, cur.nB);
        if (ok) mma_commit_elect(&bars.kempty[0]);
      }
      while (ok && cur.valid) {
        Steps nxt;
        nxt.valid = 0; nxt.nA = nxt.nB = nxt.n = 0;
        for (int j = 0; j < cur.n && ok; ++j) {
          const int gs = g + j;
          const bool last = j == cur.n - 1;
          if (last && !(ok = read_steps(kread++, nxt))) break;
          if (j < cur.nA && !(ok = issue_pv(0, gs, j == 0))) break;
          if (!last) {
            if (j + 1 < cur.nA) {
              if (!(ok = issue_s(0, gs + 1))) break;
              if (j + 1 == cur.nA - 1) mma_commit_elect(&bars.q_free[0]);
            }
          } else if (nxt.valid && !(ok = issue_s_first(0, gs + 1, nxt.nA))) {
            break;
          }
          if (j < cur.nB && !(ok = issue_pv(1, gs, j == 0))) break;
          mma_commit_elect(&bars.vempty[gs & 3]);                 // value group gs released
          if (!last) {
            if (j + 1 < cur.nB) {
              if (!(ok = issue_s(1, gs + 1))) break;
              if (j + 1 == cur.nB - 1) mma_commit_elect(&bars.q_free[1]);
            }
          } else if (nxt.valid && nxt.nB > 0 && !(ok = issue_s_first(1, gs + 1, nxt.nB))) {
            break;
          }
          if (!last || nxt.valid) mma_commit_elect(&bars.kempty[(gs + 1) & 3]);   // key group gs + 1 released
        }
        g += cur.n;
        cur = nxt;
      }
      mma_commit_elect(&bars.mma_done);     // every MMA done before TMEM is freed
      if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
      __syncwarp();
    }
  } else {
    warpgroup_reg_inc<kPrRegsSoftmax>();
    // ---------------- softmax and epilogue (warps 4-7: tile A, 8-11: tile B) ----------------
    const int x = (warp - 4) >> 2;
    const int grp = warp & 3;                     // TMEM lane quadrant of this warp
    const int row = grp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    const uint32_t tS = tmem + lane_base + (uint32_t)(x * kPrBKV);
    const uint32_t tO = tmem + lane_base + C::kOCol + (uint32_t)(x * 128);
    const float sl = p.scale_log2;
    int kread = 0;
    int ts = 0;                                   // tile-steps (s_full / pv_done phases)
    // next item in which this tile has rows
    auto next_item = [&](PairItem& it) -> bool {
      for (;;) {
        if (!pair_read_item(bars, sched_ring, kread++, lane, abort_flag, it)) return false;
        if (!it.valid || (x ? it.nB : it.nA) > 0) return true;
      }
    };
    // the previous item's output: O / row sum, bf16, row t of head h
    auto epilogue = [&](bool valid, int64_t t, int h, const uint64_t (&l2)[2]) -> bool {
      if (!mbar_wait_warp(&bars.pv_done[x], (uint32_t)(ts - 1) & 1u, abort_flag)) return false;
      tc_fence_after();
      float la, lb, lc, ld;
      f2_split(l2[0], la, lb);
      f2_split(l2[1], lc, ld);
      const float inv = (1.f / ((la + lb) + (lc + ld))) * kPrTwoMBias;
      __nv_bfloat16* dst = p.out + (t * p.H + h) * kV;
#pragma unroll
      for (int hh = 0; hh < kV / 64; ++hh) {   // 64 columns at a time: two loads in flight, one wait
        uint32_t v[64];
        tmem_ld32_nowait(tO + (uint32_t)(hh * 64), v);
        tmem_ld32_nowait(tO + (uint32_t)(hh * 64 + 32), v + 32);
        tmem_wait_ld64(v);
        if (valid) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o[e] = pack_bf16x2(__uint_as_float(v[c * 16 + 2 * e]) * inv, __uint_as_float(v[c * 16 + 2 * e + 1]) * inv);
            st_global_v8(dst + hh * 64 + c * 16, o);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.o_free[x]);
      return true;
    };

    // the item's output rows are written after the next item has been read,
    // while its first score product (whose Q needed no preparation) runs
    PairItem nxt;
    bool ok = next_item(nxt);
    bool have = false;                            // an item's output is pending
    bool prev_valid = false;
    int64_t prev_t = 0;
    int prev_h = 0;
    uint64_t l2[2] = {0ull, 0ull};                // row sum of e, as two fp32 pairs
    while (ok) {
      if (have && !(ok = epilogue(prev_valid, prev_t, prev_h, l2))) break;
      if (!nxt.valid) break;
      const PairItem cur = nxt;
      const int nX = x ? cur.nB : cur.nA;
      const int qrow = cur.q0 + x * kTile + row;  // in-sequence query index
      const bool valid = qrow < cur.L;
      const int qi = min(qrow, cur.L - 1);
      const int lim_row = cur.off + qi;             // last key this row attends
      // steps from jm on reach past the tile's first row's last key: the
      // causal mask applies there (one step without cached rows; with an
      // offset that is not a multiple of 128, two)
      const int jm = (cur.off + cur.q0 + x * kTile) / kPrBKV;
      float m = 0.f;                              // reference max (log2 units, scaled)
      l2[0] = 0ull;
      l2[1] = 0ull;
      for (int j = 0; j < nX && ok; ++j) {
        if (!mbar_wait_warp(&bars.s_full[x], (uint32_t)ts & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        // the row's 128 scores: four loads in flight, one wait
        float sc[kPrBKV];
        {
          uint32_t v[kPrBKV];
#pragma unroll
          for (int c = 0; c < kPrBKV / 32; ++c) tmem_ld32_nowait(tS + (uint32_t)(c * 32), v + c * 32);
          tmem_wait_ld128(v);
#pragma unroll
          for (int e = 0; e < kPrBKV; ++e) sc[e] = __uint_as_float(v[e]);
        }
        if (j >= jm) {            // the diagonal steps: causal mask (also masks padded keys)
          const int lim = lim_row - j * kPrBKV;
#pragma unroll
          for (int e = 0; e < kPrBKV; ++e)
            if (e > lim) sc[e] = -INFINITY;
        }
        float mx4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float a = fmax3(sc[32 * q], sc[32 * q + 1], sc[32 * q + 2]);
#pragma unroll
          for (int e = 3; e + 1 < 32; e += 2) a = fmax3(a, sc[32 * q + e], sc[32 * q + e + 1]);
          mx4[q] = fmaxf(a, sc[32 * q + 31]);
        }
        const float mx = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl;
        bool raise = false;
        if (j == 0) m = mx;
        else raise = mx > m + kPrLazy;
        if (__any_sync(0xffffffffu, raise)) {
          // rare: raise the reference; O must hold P V of every earlier step first
          if (!mbar_wait_warp(&bars.pv_done[x], (uint32_t)(ts - 1) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const float alpha = raise ? ex2_approx(m - mx) : 1.f;
          if (raise) {
            m = mx;
            const uint64_t a2 = f2_make(alpha, alpha);
            l2[0] = f2_mul(l2[0], a2);
            l2[1] = f2_mul(l2[1], a2);
          }
          for (int c = 0; c < kV / 16; ++c) {
            uint32_t v[16];
            const uint32_t ta = tO + (uint32_t)(c * 16);
            tmem_ld16(ta, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st16(ta, v);
          }
        }
        // e = 2^(s scale log2(e) - m - bias) in fp32; P's fp16 codes from e 2^-12
        const uint64_t sl2 = f2_make(sl, sl);
        const float nb = -(m + kPrBias);
        const uint64_t nb2 = f2_make(nb, nb);
        const uint64_t k12 = f2_make(kPrTwoM12, kPrTwoM12);
#pragma unroll
        for (int c = 0; c < kPrBKV / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t a = f2_fma(f2_make(sc[c * 32 + 2 * e], sc[c * 32 + 2 * e + 1]), sl2, nb2);
            float a0, a1;
            f2_split(a, a0, a1);
            const uint64_t w = f2_make(ex2_approx(a0), ex2_approx(a1));
            l2[e & 1] = f2_add(l2[e & 1], w);
            float v0, v1;
            f2_split(f2_mul(w, k12), v0, v1);
            pk[e] = f16x2_from_scaled(v0, v1);
          }
          tmem_st16(tS + (uint32_t)(c * 16), pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars.p_full[x]);
        ++ts;
      }
      if (!ok) break;
      have = true;
      prev_valid = valid;
      prev_t = cur.seq0 + qrow;
      prev_h = cur.h;
      ok = next_item(nxt);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace mla
