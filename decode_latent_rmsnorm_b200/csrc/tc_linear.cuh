// Tensor-core (tcgen05) Linear for the projections on either side of the
// path: out[t, j] = sum_k x[t, k] w[j, k] (nn.Linear without bias, weight
// [Nout, K]).
//
// Sources: Kimi-K2 "RoPE coefficients" page, "Query heads" (mla-init,
// mla-queries: q_a_proj, q_b_proj) and "Key heads" (mla-kv:
// kv_a_proj_with_mqa); GLM-5 "Normalized key-value latent" page,
// "Key-value compression" (the same Linears, and o_proj).
//
// One CTA computes a tile of 128 rows of x (M of the MMA, TMEM lane = row)
// by kBN output features (N, 128..256), over one K split: stages of 64 K
// values, x box [128 rows x 64] and weight box [kBN rows x 64], both K-major
// with the 128-byte swizzle, as many stages in flight as shared memory holds
// (up to six). An M128 x N(kBN) product
// reads 4 KB of x and kBN / 8 KB of weight per 16 K values, within the SM's
// shared-memory bandwidth for kBN >= 128. With splits > 1 each CTA covers
// its share of the K stages and writes an fp32 partial [split][n][Nout]; the
// kernel that consumes the result adds the partials in split order (fixed
// order: the sums do not depend on scheduling). With one split the result is
// written in fp32 (out_f32) or bf16 (out).
// Warps: 0 TMA, 1 MMA (whole warp, one elected lane issues), 2-5 epilogue
// (warp w reads TMEM lanes 32 (w % 4) ..).
#pragma once
#include "tc_ptx.cuh"

namespace mla {
namespace tc {

constexpr int kLinThreads = 192;
constexpr int kLinABytes = 128 * 128;   // 128 rows x 64 K, 16-bit

template <int kBN>
struct LinCfg {
  static constexpr int kBBytes = kBN * 128;
  static constexpr int kFit = (232448 - 1024) / (kLinABytes + kBBytes);
  static constexpr int kStages = kFit < 6 ? kFit : 6;
  static constexpr size_t kSmem = (size_t)kStages * (kLinABytes + kBBytes) + 1024;
  static constexpr uint32_t kTmemCols = 256;
  static_assert(kBN % 32 == 0 && kBN >= 128 && kBN <= 256, "N of the product: 128..256, a multiple of 32");
  static_assert(kSmem <= 232448, "stages exceed shared memory");
};

struct LinParams {
  int64_t n;            // rows of x
  int K, Nout;          // K a multiple of 64; Nout a multiple of 32
  int splits;           // K splits (grid z)
  __nv_bfloat16* out;   // [n, Nout] bf16 (splits == 1, out_f32 == nullptr)
  float* out_f32;       // [splits, n, Nout] fp32 partials, or the fp32 result when splits == 1
};

template <int kBN, bool kF16>
__global__ void __launch_bounds__(kLinThreads, 1)
linear_tc_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                 LinParams p) {
  using C = LinCfg<kBN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  constexpr int kLinStages = C::kStages;
  __shared__ uint64_t full[kLinStages], empty[kLinStages], done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_allow_next();   // the kernel that reads the result may start its own preparation
  const int n0 = blockIdx.x * kBN;                    // first output feature
  const int64_t m0 = (int64_t)blockIdx.y * 128;       // first row of x
  const int ks = blockIdx.z;
  const int ns = p.K / 64;
  const int s0 = (int)((int64_t)ks * ns / p.splits), s1 = (int)((int64_t)(ks + 1) * ns / p.splits);
  const int nk = s1 - s0;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kLinStages * kLinABytes;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kLinStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(&done, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&map_x);
      tma_prefetch_desc(&map_w);
      bool ok = true;
      int kc = 0;
      for (; kc < nk; ++kc) {
        const int s = kc % kLinStages;
        if (kc >= kLinStages &&
            !mbar_wait(&empty[s], ((uint32_t)(kc / kLinStages) & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[s], kLinABytes + C::kBBytes);
        tma_load_2d(sA + s * kLinABytes, &map_x, &full[s], (s0 + kc) * 64, (int)m0);
        tma_load_2d(sB + s * C::kBBytes, &map_w, &full[s], (s0 + kc) * 64, n0);
      }
      if (!ok)   // let the copies already issued land before the CTA exits
        for (int i = (kc > kLinStages ? kc - kLinStages : 0); i < kc; ++i)
          mbar_wait_drain(&full[i % kLinStages], (uint32_t)(i / kLinStages) & 1u);
    }
  } else if (warp == 1) {
    const uint32_t idesc = kF16 ? idesc_f16_f32(128, kBN) : idesc_bf16_f32(128, kBN);
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % kLinStages;
      if (!mbar_wait_warp(&full[s], (uint32_t)(kc / kLinStages) & 1u, &abort_flag)) break;
      tc_fence_after();
      const uint64_t ad = desc_kmajor_sw128(smem_u32(sA + s * kLinABytes));
      const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + s * C::kBBytes));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_ss_elect(tmem, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kc | k) != 0);
      mma_commit_elect(&empty[s]);
    }
    mma_commit_elect(&done);
    if (lane == 0) mbar_wait_drain(&done, 0);
    __syncwarp();
  } else {
    const int grp = warp & 3;
    const int64_t row = m0 + grp * 32 + lane;
    const bool live = row < p.n && nk > 0;
    if (mbar_wait_warp(&done, 0, &abort_flag)) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(grp * 32) << 16) + (uint32_t)(c * 32), v);
        const int col = n0 + c * 32;
        if (!live || col >= p.Nout) continue;
        if (p.out_f32) {
          uint4* dst = reinterpret_cast<uint4*>(p.out_f32 + ((int64_t)ks * p.n + row) * p.Nout + col);
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(p.out + row * p.Nout + col);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * e]), __uint_as_float(v[8 * e + 1])),
                                pack_bf16x2(__uint_as_float(v[8 * e + 2]), __uint_as_float(v[8 * e + 3])),
                                pack_bf16x2(__uint_as_float(v[8 * e + 4]), __uint_as_float(v[8 * e + 5])),
                                pack_bf16x2(__uint_as_float(v[8 * e + 6]), __uint_as_float(v[8 * e + 7])));
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
