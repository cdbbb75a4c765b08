// Tensor-core (tcgen05) causal attention, two query tiles per CTA.
//
// Sources: Kimi-K2 "Query content heads" page, "Join query parts", and the
// Kimi-K2 "RoPE coefficients" page, "Key heads" (mla-prefill excerpt): each
// head's query and key join their non-rotary and rotary parts (the key's
// rotary part is the one rotary key shared by all heads), the scores are
// scaled, causally masked, normalized with a softmax in fp32 and mix the
// values. The arithmetic is the one of attention_kernel; this kernel changes
// how it is scheduled on the SM.
//
// One CTA = one head x one 256-row block of queries, split into tile A (rows
// 0-127) and tile B (rows 128-255). Both tiles read the same key / value
// tiles (128 keys per step), so each K/V byte staged in shared memory feeds
// twice the tensor-core work. Warps:
//   warp 0     TMA producer (Q tiles, then per step: the key atoms and the two
//              transposed value boxes into a ring of 16 KB slots)
//   warp 1     MMA issuer (whole warp, one elected lane issues)
//   warps 2-5  softmax of tile A (one query row per thread, TMEM lane = row)
//   warps 6-9  softmax of tile B
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,256+V),
// O_B [384,384+V). P (fp16) is written back over the first 64 columns of its
// own S buffer and read from there by the P V product (A operand in TMEM).
// The MMA thread alternates the tiles so that one tile's softmax runs while
// the tensor cores work on the other tile:
//   ... PV_A(j)  S_A(j+1)  PV_B(j)  S_B(j+1)  PV_A(j+1) ...
// Tensor-core instructions from one thread run in issue order, so S_X(j+1)
// overwrites P_X(j) only after PV_X(j) has read it.
//
// Softmax reference: a row's reference m is its maximum over the first key
// tile; it is raised (and O and the row sum rescaled) only when a later tile's
// maximum exceeds it by more than kPrLazy (log2 units), so P <= 2^kPrLazy,
// well inside fp16. The row sum adds the fp32 weights before their rounding
// to fp16 (relative difference <= 2^-12 of the result).
#pragma once
#include "tc_attention.cuh"

namespace mla {
namespace tc {

constexpr int kPrBKV = 128;                 // keys per step
constexpr int kPrThreads = 320;
constexpr int kPrSlotBytes = 16384;
constexpr int kPrMaxSlots = 12;
constexpr float kPrLazy = 8.f;
constexpr int kPrGroupDepth = 4;

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
// once per box. The barriers rotate over kPrGroupDepth steps: a box's slot
// was last used at most three steps earlier (static_assert below), and the
// release the producer waits for before re-arming a step's barrier is issued
// after the MMA warp's wait on that barrier four steps earlier.
struct PairBarriers {
  uint64_t q_full, q_ready[2];
  uint64_t kfull[kPrGroupDepth], kempty[kPrGroupDepth], vfull[kPrGroupDepth], vempty[kPrGroupDepth];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

template <int kN, int kV>
__global__ void __launch_bounds__(kPrThreads, 1)
attention_pair_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kn,
                      const __grid_constant__ CUtensorMap map_kr, const __grid_constant__ CUtensorMap map_vt,
                      AttParams p) {
  using C = PairCfg<kN, kV>;
  constexpr int S = C::kSlots;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ PairBarriers bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_allow_next();
  const int rank = blockIdx.x / p.H, h = blockIdx.x % p.H;
  const int tile = p.order[rank];       // first tile of the block
  if (tile < 0) return;                 // uniform over the CTA
  const int seq = p.tile_seq[tile];
  const int q0 = p.tile_q0[tile];       // multiple of 256
  const int64_t seq0 = p.cu[seq];
  const int L = (int)(p.cu[seq + 1] - seq0);
  const int kv_pad0 = p.seq_tile0[seq] * kTile;
  const int nA = q0 / kPrBKV + 1;                              // key steps of tile A
  const int nB = (q0 + kTile < L) ? q0 / kPrBKV + 2 : 0;      // 0: tile B is all padding
  const int n = nA > nB ? nA : nB;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sRing = smem + C::kQBytes;
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars.q_ready[x], 128);
      mbar_init(&bars.s_full[x], 1);
      mbar_init(&bars.p_full[x], 128);
      mbar_init(&bars.pv_done[x], 1);
    }
    for (int b = 0; b < kPrGroupDepth; ++b) {
      mbar_init(&bars.kfull[b], 1); mbar_init(&bars.kempty[b], 1);
      mbar_init(&bars.vfull[b], 1); mbar_init(&bars.vempty[b], 1);
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

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_kn);
      tma_prefetch_desc(&map_kr);
      tma_prefetch_desc(&map_vt);
      mbar_arrive_expect_tx(&bars.q_full, nB > 0 ? C::kQBytes : C::kQTileBytes);
      for (int a = 0; a < C::kQAtoms; ++a)
        tma_load_3d(sQ + a * kTile * 128, &map_q, &bars.q_full, a * 64, h, (int)(seq0 + q0));
      if (nB > 0)
        for (int a = 0; a < C::kQAtoms; ++a)
          tma_load_3d(sQ + C::kQTileBytes + a * kTile * 128, &map_q, &bars.q_full, a * 64, h,
                      (int)(seq0 + q0 + kTile));
      // box g of the ring sits in slot g % S; before it is filled, the group
      // that last used the slot (box g - S) must have been released
      auto wait_released = [&](int gp) -> bool {
        const int jp = gp / C::kBoxes;
        uint64_t* bar = (gp % C::kBoxes) < C::kQAtoms ? &bars.kempty[jp & 3] : &bars.vempty[jp & 3];
        return mbar_wait(bar, (uint32_t)(jp >> 2) & 1u, abort_flag);
      };
      pdl_wait();   // k_nope, the values and k_rot come from the previous kernel
      bool ok = true;
      int jk = -1, jv = -1;              // last key / value group issued
      for (int j = 0; j < n && ok; ++j) {
        const int kv_row = kv_pad0 + j * kPrBKV;
        const int g0 = j * C::kBoxes;
        for (int i = 0; i < C::kQAtoms && ok; ++i)
          if (g0 + i >= S) ok = wait_released(g0 + i - S);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.kfull[j & 3], C::kQAtoms * kPrBKV * 128);
        for (int i = 0; i < C::kKAtoms; ++i)
          tma_load_2d(sRing + ((g0 + i) % S) * kPrSlotBytes, &map_kn, &bars.kfull[j & 3], i * 64,
                      h * p.Tpad + kv_row);
        tma_load_2d(sRing + ((g0 + C::kKAtoms) % S) * kPrSlotBytes, &map_kr, &bars.kfull[j & 3], 0, kv_row);
        jk = j;
        for (int v = 0; v < 2 && ok; ++v)
          if (g0 + C::kQAtoms + v >= S) ok = wait_released(g0 + C::kQAtoms + v - S);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars.vfull[j & 3], 2 * C::kVBoxBytes);
        for (int v = 0; v < 2; ++v)
          tma_load_2d(sRing + ((g0 + C::kQAtoms + v) % S) * kPrSlotBytes, &map_vt, &bars.vfull[j & 3],
                      kv_row + v * 64, h * kV);
        jv = j;
      }
      if (!ok) {   // let every copy already issued land before the CTA exits
        mbar_wait_drain(&bars.q_full, 0);
        for (int jj = (jk > 3 ? jk - 3 : 0); jj <= jk; ++jj)
          mbar_wait_drain(&bars.kfull[jj & 3], (uint32_t)(jj >> 2) & 1u);
        for (int jj = (jv > 3 ? jv - 3 : 0); jj <= jv; ++jj)
          mbar_wait_drain(&bars.vfull[jj & 3], (uint32_t)(jj >> 2) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    const uint32_t idesc_s = idesc_f16_f32(kTile, kPrBKV);
    const uint32_t idesc_o = idesc_f16_f32(kTile, kV);
    auto slot_addr = [&](int g) -> uint32_t { return smem_u32(sRing + (g % S) * kPrSlotBytes); };
    int k_seen = -1, v_seen = -1;        // last step whose key / value group was waited for
    // S_x(j) = Q_x K_j^T over all D columns
    auto issue_s = [&](int x, int j) -> bool {
      if (k_seen < j) {
        if (!mbar_wait_warp(&bars.kfull[j & 3], (uint32_t)(j >> 2) & 1u, abort_flag)) return false;
        k_seen = j;
      }
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(x * kPrBKV);
#pragma unroll
      for (int a = 0; a < C::kQAtoms; ++a) {
        const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + x * C::kQTileBytes + a * kTile * 128));
        const uint64_t kd = desc_kmajor_sw128(slot_addr(j * C::kBoxes + a));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ss_elect(d, desc_advance(qd, k * 32), desc_advance(kd, k * 32), idesc_s, (a | k) != 0);
      }
      mma_commit_elect(&bars.s_full[x]);
      return true;
    };
    // O_x += P_x(j) V_j, P_x(j) read from TMEM
    auto issue_pv = [&](int x, int j) -> bool {
      if (v_seen < j) {
        if (!mbar_wait_warp(&bars.vfull[j & 3], (uint32_t)(j >> 2) & 1u, abort_flag)) return false;
        v_seen = j;
      }
      if (!mbar_wait_warp(&bars.p_full[x], (uint32_t)j & 1u, abort_flag)) return false;
      tc_fence_after();
      const uint32_t pa = tmem + (uint32_t)(x * kPrBKV);
      const uint32_t o = tmem + C::kOCol + (uint32_t)(x * 128);
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const uint64_t vd = desc_kmajor_sw128(slot_addr(j * C::kBoxes + C::kQAtoms + v));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ts_elect(o, pa + (uint32_t)((v * 4 + k) * 8), desc_advance(vd, k * 32), idesc_o, (j | v | k) != 0);
      }
      mma_commit_elect(&bars.pv_done[x]);
      return true;
    };

    bool ok = mbar_wait_warp(&bars.q_ready[0], 0, abort_flag);
    if (ok && nB > 0) ok = mbar_wait_warp(&bars.q_ready[1], 0, abort_flag);
    if (ok) ok = issue_s(0, 0);
    if (ok && nB > 0) ok = issue_s(1, 0);
    if (ok) mma_commit_elect(&bars.kempty[0]);
    for (int j = 0; j < n && ok; ++j) {
      const bool a_now = j < nA, b_now = j < nB, a_next = j + 1 < nA, b_next = j + 1 < nB;
      if (a_now && !(ok = issue_pv(0, j))) break;
      if (a_next && !(ok = issue_s(0, j + 1))) break;
      if (b_now && !(ok = issue_pv(1, j))) break;
      mma_commit_elect(&bars.vempty[j & 3]);                 // value group j released
      if (b_next && !(ok = issue_s(1, j + 1))) break;
      if (a_next || b_next) mma_commit_elect(&bars.kempty[(j + 1) & 3]);   // key group j + 1 released
    }
    mma_commit_elect(&bars.mma_done);     // every MMA done before TMEM is freed
    if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
    __syncwarp();
  } else {
    // ---------------- softmax and epilogue (warps 2-5: tile A, 6-9: tile B) ----------------
    const int x = (warp - 2) >> 2;
    const int nX = x ? nB : nA;
    const int grp = warp & 3;                     // TMEM lane quadrant of this warp
    const int row = grp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    const int qrow = q0 + x * kTile + row;        // in-sequence query index
    const bool valid = qrow < L;
    const int qi = min(qrow, L - 1);
    const int64_t t = seq0 + qrow;
    bool ok = nX > 0;
    if (ok) ok = mbar_wait_warp(&bars.q_full, 0, abort_flag);
    if (ok) {
      // this row of q: bf16 -> fp16 in place (per atom: all loads, the
      // conversion, then all stores); the rotary atom is rotated at the
      // token's position, its 32 pairs in two halves of 16
      uint8_t* sQx = sQ + x * C::kQTileBytes;
      float qmax = 0.f;
#pragma unroll 1
      for (int a = 0; a < C::kQAtoms - 1; ++a) {
        uint8_t* qa = sQx + a * kTile * 128;
        uint4 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = *reinterpret_cast<const uint4*>(qa + sw128_offset(row, c));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t w4[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
          uint32_t o4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w4[e]);
            qmax = fmaxf(qmax, fmaxf(fabsf(f.x), fabsf(f.y)));
            o4[e] = pack_f16x2(f.x, f.y);
          }
          v[c] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(qa + sw128_offset(row, c)) = v[c];
      }
      const int64_t pos = valid ? checked_pos(p.positions[t], p.max_pos) : 0;
      uint8_t* qr = sQx + (C::kQAtoms - 1) * kTile * 128;
#pragma unroll 1
      for (int hp = 0; hp < 2; ++hp) {
        // rotary pairs [16 hp, 16 hp + 16): 16 cos / sin entries as four vector
        // loads each; the four 16-byte chunks holding the pairs' 32 values
        // (half-split pairing: chunks 2hp, 2hp+1 and 4+2hp, 5+2hp;
        // interleaved: chunks 4hp .. 4hp+3)
        const float4* c4 = reinterpret_cast<const float4*>(p.cos_t + pos * 32 + hp * 16);
        const float4* s4 = reinterpret_cast<const float4*>(p.sin_t + pos * 32 + hp * 16);
        float cs[16], sn[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 cv = c4[i], sv = s4[i];
          cs[4 * i] = cv.x; cs[4 * i + 1] = cv.y; cs[4 * i + 2] = cv.z; cs[4 * i + 3] = cv.w;
          sn[4 * i] = sv.x; sn[4 * i + 1] = sv.y; sn[4 * i + 2] = sv.z; sn[4 * i + 3] = sv.w;
        }
        int ch[4];
        if (p.interleaved) {
          ch[0] = 4 * hp; ch[1] = 4 * hp + 1; ch[2] = 4 * hp + 2; ch[3] = 4 * hp + 3;
        } else {
          ch[0] = 2 * hp; ch[1] = 2 * hp + 1; ch[2] = 4 + 2 * hp; ch[3] = 5 + 2 * hp;
        }
        float xr[32];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 v = *reinterpret_cast<const uint4*>(qr + sw128_offset(row, ch[k]));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w4[e]);
            xr[k * 8 + 2 * e] = f.x;
            xr[k * 8 + 2 * e + 1] = f.y;
          }
        }
        // xr holds, in order, chunks ch[0..3]; local pair i is (xr[2i],
        // xr[2i+1]) when interleaved, (xr[i], xr[16+i]) otherwise
        float y[32];
        if (p.interleaved) {
#pragma unroll
          for (int i = 0; i < 16; ++i) rope_turn(xr[2 * i], xr[2 * i + 1], cs[i], sn[i], y[2 * i], y[2 * i + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) rope_turn(xr[i], xr[16 + i], cs[i], sn[i], y[i], y[16 + i]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 v;
          v.x = pack_f16x2(y[k * 8 + 0], y[k * 8 + 1]);
          v.y = pack_f16x2(y[k * 8 + 2], y[k * 8 + 3]);
          v.z = pack_f16x2(y[k * 8 + 4], y[k * 8 + 5]);
          v.w = pack_f16x2(y[k * 8 + 6], y[k * 8 + 7]);
          *reinterpret_cast<uint4*>(qr + sw128_offset(row, ch[k])) = v;
#pragma unroll
          for (int e = 0; e < 8; ++e) qmax = fmaxf(qmax, fabsf(y[k * 8 + e]));
        }
      }
      if (valid && !(qmax <= kF16Max)) raise_device_error(kDevErrRange);
      fence_proxy_async_smem();
      mbar_arrive(&bars.q_ready[x]);
    }

    const uint32_t tS = tmem + lane_base + (uint32_t)(x * kPrBKV);
    const uint32_t tO = tmem + lane_base + C::kOCol + (uint32_t)(x * 128);
    const float sl = p.scale_log2;
    float m = 0.f;            // reference max (log2 units, scaled)
    float l = 0.f;            // running sum of the weights at that reference
    for (int j = 0; j < nX && ok; ++j) {
      if (!mbar_wait_warp(&bars.s_full[x], (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
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
      if (j == nX - 1) {        // the diagonal step: causal mask (also masks padded keys)
        const int lim = qi - j * kPrBKV;
#pragma unroll
        for (int e = 0; e < kPrBKV; ++e)
          if (e > lim) sc[e] = -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int e = 0; e < kPrBKV; ++e) mx4[e & 3] = fmaxf(mx4[e & 3], sc[e]);
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * sl;
      bool raise = false;
      if (j == 0) m = mx;
      else raise = mx > m + kPrLazy;
      if (__any_sync(0xffffffffu, raise)) {
        // rare: raise the reference; O must hold P V of every earlier step first
        if (!mbar_wait_warp(&bars.pv_done[x], (uint32_t)(j - 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const float alpha = raise ? ex2_approx(m - mx) : 1.f;
        if (raise) { m = mx; l *= alpha; }
        for (int c = 0; c < kV / 16; ++c) {
          uint32_t v[16];
          const uint32_t ta = tO + (uint32_t)(c * 16);
          tmem_ld16(ta, v);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st16(ta, v);
        }
      }
      // P = 2^(s scale log2(e) - m) in fp32, packed to fp16; the row sum adds
      // the fp32 weights before their rounding to fp16.
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kPrBKV / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a0 = fmaf(sc[c * 32 + 2 * e], sl, -m);
          const float a1 = fmaf(sc[c * 32 + 2 * e + 1], sl, -m);
          const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
          rs4[e & 3] += p0 + p1;
          pk[e] = pack_f16x2(p0, p1);
        }
        tmem_st16(tS + (uint32_t)(c * 16), pk);
      }
      l += (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars.p_full[x]);
    }
    if (ok && nX > 0) ok = mbar_wait_warp(&bars.pv_done[x], (uint32_t)(nX - 1) & 1u, abort_flag);
    if (ok && nX > 0) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* dst = p.out + (t * p.H + h) * kV;
      for (int c = 0; c < kV / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(tO + (uint32_t)(c * 16), v);
        if (valid) {
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            o[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 16);
          d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
          d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
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
