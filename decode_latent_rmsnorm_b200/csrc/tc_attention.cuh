// Tensor-core (tcgen05) causal attention over the padded k_nope / transposed
// value / rotated k_rot workspace written by norm_kvb_gemm_kernel.
//
// Sources: Kimi-K2 "Query content heads" page, "Join query parts" and the
// Kimi-K2 "RoPE coefficients" page, "Key heads" (mla-prefill excerpt): the
// rotary parts are rotated; each head's query and key join their non-rotary
// and rotary parts, the key's rotary part being the one shared rotary key;
// scores are scaled, causally masked, normalized with a softmax in fp32 and
// used to mix the values.
//
// Operands: the non-rotary score atoms multiply q as given (bf16) with k_nope
// in bf16; the rotary atom multiplies q's rotary part, rotated once per row
// by the preparation kernel, with the rotated shared key, both fp16; P and
// the values are fp16; accumulators fp32, output bf16. Q therefore needs no
// work on the SM: the first score product starts when its copy lands.
//
// One CTA = one (128-query tile, head). Warp 0 issues TMA loads, warp 1 issues
// the MMAs, warps 2-5 own one query row per thread (TMEM lane = row):
//   S_j   = Q K_j^T           (tcgen05, fp32 in TMEM, double buffered)
//   P_j   = exp2(S_j * scale * log2 e - m)   (online softmax, registers; fp16
//           P written back over S_j in TMEM)
//   O    += P_j V_j           (tcgen05, P read from TMEM, fp32 accumulator)
// With P in TMEM and S double-buffered, the softmax of step j + 1 does not
// wait for the P V product of step j. The shared rotary key tile is loaded
// once per key tile and serves every query row of the head. The reference m
// of a row is raised only when a score exceeds it by more than kAttLazy
// (log2 units; P <= 2^kAttLazy stays well inside fp16), and O is rescaled
// (in TMEM, by the softmax warps) only then.
#pragma once
#include "tc_gemm.cuh"

namespace mla {
namespace tc {

constexpr int kAttBKV = 64;                       // keys per tile (MMA N of S, K of PV)
constexpr int kAttThreads = 192;
constexpr float kAttLazy = 8.f;                   // reference max slack (log2 units)

template <int kN, int kV, int kStages>
struct AttCfg {
  static constexpr int D = kN + 64;
  static constexpr int kQAtoms = D / 64;
  static constexpr int kQBytes = kQAtoms * kTile * 128;
  static constexpr int kKAtomBytes = kAttBKV * 128;
  static constexpr int kKBytes = kQAtoms * kKAtomBytes;
  static constexpr int kVBytes = kV * 128;         // [kV rows x 64 keys]
  static constexpr int kStageBytes = kKBytes + kVBytes;
  static constexpr size_t kSmem = (size_t)kQBytes + (size_t)kStages * kStageBytes + 1024;
  static constexpr int kSCol = 0;                  // S buffers: columns [0, 128)
  static constexpr int kOCol = 2 * kAttBKV;        // O: columns [128, 128 + kV)
  static constexpr uint32_t kTmemCols = (kOCol + kV) <= 256 ? 256 : 512;
};

struct AttParams {
  const int32_t* cu;
  const int32_t* positions;
  const int32_t* seq_tile0;
  const int32_t* tile_seq;
  const int32_t* tile_q0;
  const int32_t* order;
  const float* cos_t;
  const float* sin_t;
  __nv_bfloat16* out;
  int* item_counter;            // two-tile kernel: next work item (zeroed by the preparation kernel)
  const int32_t* q_off;         // two-tile kernel: per sequence, the key index of its first query
                                // (cached rows before it; NULL: 0). Keys come from the padded
                                // layout of the sequence's q_off + length rows.
  int H, Tpad, max_pos, interleaved;
  int n_blocks;                 // two-tile kernel: entries of `order` (256-row blocks, -1 past the last)
  float scale_log2;             // softmax scale * log2(e)
};

template <int kStages>
struct AttBarriers {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];              // P of the step in S buffer b written (TMEM)
  uint64_t pv_done[2], mma_done;   // pv_done[j & 1]: the P V product of step j
  uint32_t tmem_base;
  int abort_flag;
};

template <int kN, int kV, int kStages>
__global__ void __launch_bounds__(kAttThreads, 1)
attention_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_qr,
                 const __grid_constant__ CUtensorMap map_kn, const __grid_constant__ CUtensorMap map_kr,
                 const __grid_constant__ CUtensorMap map_vt, AttParams p) {
  using C = AttCfg<kN, kV, kStages>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ AttBarriers<kStages> bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_allow_next();
  // head-major grid: the CTAs that run at the same time share a head's keys
  // and values, which stay in L2 (heads interleaved, every CTA streamed its
  // keys and values from DRAM); within a head, heaviest tiles first
  const int n_rank = (int)gridDim.x / p.H;
  const int rank = (int)blockIdx.x % n_rank, h = (int)blockIdx.x / n_rank;
  const int tile = p.order[rank];
  if (tile < 0) return;   // uniform over the CTA
  const int seq = p.tile_seq[tile];
  const int q0 = p.tile_q0[tile];
  const int64_t seq0 = p.cu[seq];
  const int L = (int)(p.cu[seq + 1] - seq0);
  const int kv_pad0 = p.seq_tile0[seq] * kTile;           // padded row of key 0
  const int kv_len = min(L, q0 + kTile);
  const int n_kv = (kv_len + kAttBKV - 1) / kAttBKV;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&bars.kv_full[s], 1); mbar_init(&bars.kv_empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&bars.s_full[b], 1); mbar_init(&bars.s_free[b], 128); }
    for (int b = 0; b < 2; ++b) mbar_init(&bars.p_full[b], 128);
    mbar_init(&bars.pv_done[0], 1);
    mbar_init(&bars.pv_done[1], 1);
    mbar_init(&bars.mma_done, 1);
    bars.abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&bars.tmem_base, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_qr);
      tma_prefetch_desc(&map_kn);
      tma_prefetch_desc(&map_kr);
      tma_prefetch_desc(&map_vt);
      // Q's non-rotary atoms as given (bf16) and its rotary atom rotated by the
      // preparation kernel (fp16; that kernel finished before the previous one
      // started)
      mbar_arrive_expect_tx(&bars.q_full, C::kQBytes);
      for (int a = 0; a < kN / 64; ++a)
        tma_load_3d(sQ + a * kTile * 128, &map_q, &bars.q_full, a * 64, h, (int)(seq0 + q0));
      tma_load_3d(sQ + (kN / 64) * kTile * 128, &map_qr, &bars.q_full, 0, h, (int)(seq0 + q0));
      pdl_wait();   // k_nope, the values and k_rot come from the previous kernel
      bool ok = true;
      int j = 0;
      for (; j < n_kv; ++j) {
        const int s = j % kStages;
        if (!mbar_wait(&bars.kv_empty[s], ((uint32_t)(j / kStages) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* sK = sKV + s * C::kStageBytes;
        uint8_t* sV = sK + C::kKBytes;
        const int kv_row = kv_pad0 + j * kAttBKV;
        mbar_arrive_expect_tx(&bars.kv_full[s], C::kStageBytes);
        for (int a = 0; a < kN / 64; ++a)
          tma_load_2d(sK + a * C::kKAtomBytes, &map_kn, &bars.kv_full[s], a * 64, h * p.Tpad + kv_row);
        tma_load_2d(sK + (kN / 64) * C::kKAtomBytes, &map_kr, &bars.kv_full[s], 0, kv_row);
        tma_load_2d(sV, &map_vt, &bars.kv_full[s], kv_row, h * kV);
      }
      if (!ok) {   // let every copy already issued land before the CTA exits
        mbar_wait_drain(&bars.q_full, 0);
        for (int i = (j > kStages ? j - kStages : 0); i < j; ++i)
          mbar_wait_drain(&bars.kv_full[i % kStages], (uint32_t)(i / kStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    const uint32_t idesc_s_nope = idesc_bf16_f32(kTile, kAttBKV);   // q as given, k_nope in bf16
    const uint32_t idesc_s_rope = idesc_f16_f32(kTile, kAttBKV);    // rotated q and key in fp16
    const uint32_t idesc_o = idesc_f16_f32(kTile, kV);
    const uint32_t o_tmem = tmem + C::kOCol;
    bool ok = mbar_wait_warp(&bars.q_full, 0, abort_flag);
    tc_fence_after();
    auto issue_pv = [&](int jj) -> bool {
      if (!mbar_wait_warp(&bars.p_full[jj & 1], (uint32_t)(jj >> 1) & 1u, abort_flag)) return false;
      tc_fence_after();
      const int s = jj % kStages;
      const uint32_t pa = tmem + C::kSCol + (uint32_t)((jj & 1) * kAttBKV);   // P over S_jj, 8 columns per 16 keys
      const uint64_t vd = desc_kmajor_sw128(smem_u32(sKV + s * C::kStageBytes + C::kKBytes));
#pragma unroll
      for (int k = 0; k < kAttBKV / 16; ++k)
        mma_ts_elect(o_tmem, pa + (uint32_t)(k * 8), desc_advance(vd, k * 32), idesc_o, (jj | k) != 0);
      mma_commit_elect(&bars.kv_empty[s]);
      mma_commit_elect(&bars.pv_done[jj & 1]);
      return true;
    };
    for (int j = 0; j < n_kv && ok; ++j) {
      const int s = j % kStages, b = j & 1;
      if (!mbar_wait_warp(&bars.kv_full[s], (uint32_t)(j / kStages) & 1u, abort_flag)) { ok = false; break; }
      if (!mbar_wait_warp(&bars.s_free[b], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint8_t* sK = sKV + s * C::kStageBytes;
      const uint32_t s_tmem = tmem + C::kSCol + b * kAttBKV;
#pragma unroll
      for (int a = 0; a < C::kQAtoms; ++a) {
        const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + a * kTile * 128));
        const uint64_t kd = desc_kmajor_sw128(smem_u32(sK + a * C::kKAtomBytes));
        const uint32_t idesc_s = a < kN / 64 ? idesc_s_nope : idesc_s_rope;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ss_elect(s_tmem, desc_advance(qd, k * 32), desc_advance(kd, k * 32), idesc_s, (a | k) != 0);
      }
      mma_commit_elect(&bars.s_full[b]);
      if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok && n_kv > 0) issue_pv(n_kv - 1);
    mma_commit_elect(&bars.mma_done);     // every MMA done before TMEM is freed
    if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
    __syncwarp();
  } else {
    // ---------------- softmax / correction / epilogue (warps 2-5) ----------------
    const int grp = warp & 3;
    const int row = grp * 32 + lane;
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    const bool valid = (q0 + row) < L;
    const int qi = min(q0 + row, L - 1);          // in-sequence query index used by the mask
    const int64_t t = seq0 + q0 + row;
    bool ok = true;

    float m = -INFINITY;      // running max (log2 units) used as the exponent's reference
    float l = 0.f;            // running sum of P at that reference
    for (int j = 0; j < n_kv && ok; ++j) {
      const int b = j & 1;
      if (!mbar_wait_warp(&bars.s_full[b], (uint32_t)(j >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sc[kAttBKV];
#pragma unroll
      for (int c = 0; c < kAttBKV / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(C::kSCol + b * kAttBKV + c * 16), v);
#pragma unroll
        for (int e = 0; e < 16; ++e) sc[c * 16 + e] = __uint_as_float(v[e]);
      }
      tc_fence_before();
      mbar_arrive(&bars.s_free[b]);
      const int kv0 = j * kAttBKV;
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < kAttBKV; ++e) {
        const float v = (kv0 + e <= qi) ? sc[e] * p.scale_log2 : -INFINITY;   // causal mask
        sc[e] = v;
        mx = fmaxf(mx, v);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mx > m + kAttLazy) {
        if (m != -INFINITY) { alpha = ex2_approx(m - mx); rescale = true; }
        m = mx;
      }
      float rs = 0.f;
      uint32_t pk[kAttBKV / 2];
#pragma unroll
      for (int e = 0; e < kAttBKV; e += 2) {
        const float p0 = ex2_approx(sc[e] - m), p1 = ex2_approx(sc[e + 1] - m);
        pk[e / 2] = pack_f16x2(p0, p1);
        // the row sum uses the same rounded weights the P V product sees, so
        // the output is an exact convex combination of those weights
        const float2 pr = unpack_f16x2(pk[e / 2]);
        rs += pr.x + pr.y;
      }
      l = l * alpha + rs;
      if (j >= 1 && __any_sync(0xffffffffu, rescale)) {   // warp-collective TMEM access: whole warp, alpha = 1 elsewhere
        // O is stable once the P V product of step j - 1 is done (that of
        // step j - 2 is: S_j was issued after it; step j + 1's is not issued)
        if (!mbar_wait_warp(&bars.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          for (int c = 0; c < kV / 16; ++c) {
            uint32_t v[16];
            const uint32_t ta = tmem + lane_base + (uint32_t)(C::kOCol + c * 16);
            tmem_ld16(ta, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st16(ta, v);
          }
          tmem_st_wait();
        }
      }
      // P over this step's S columns (this thread's lane; its scores are read)
      {
        const uint32_t tp = tmem + lane_base + (uint32_t)(C::kSCol + b * kAttBKV);
        uint32_t h0[16], h1[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) { h0[e] = pk[e]; h1[e] = pk[16 + e]; }
        tmem_st16(tp, h0);
        tmem_st16(tp + 16, h1);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&bars.p_full[b]);
    }
    // the last two P V products, each on the barrier of its step's parity
    // (the previous phase of either is complete and no later one is issued,
    // so each wait is at most one phase behind)
    if (ok && n_kv > 1)
      ok = mbar_wait_warp(&bars.pv_done[(n_kv - 2) & 1], (uint32_t)((n_kv - 2) >> 1) & 1u, abort_flag);
    if (ok && n_kv > 0)
      ok = mbar_wait_warp(&bars.pv_done[(n_kv - 1) & 1], (uint32_t)((n_kv - 1) >> 1) & 1u, abort_flag);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* dst = p.out + (t * p.H + h) * kV;
      for (int c = 0; c < kV / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(C::kOCol + c * 16), v);
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
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace tc
}  // namespace mla
