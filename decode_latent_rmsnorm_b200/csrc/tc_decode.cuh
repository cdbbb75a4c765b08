// Absorbed MLA decode over the latent cache on tensor cores (tcgen05).
//
// Sources: GLM-5 "Normalized key-value latent" page, "KV cache" (the cache
// holds the normalized latent and the rotated shared key; heads are expanded
// from every cached row) and the "Eager latent expansion" equation page,
// "Read the equation" (the absorbed path contracts the projection weights
// with the queries and with the latent aggregate instead of expanding K/V).
//
// Per sequence b and head h, with W_UK_h / W_UV_h the k_nope / value rows of
// head h in kv_b_proj:
//   q_lat = W_UK_h^T q_nope,  q_pe' = rope(q_pe, pos_b)          (qprep)
//   s_t   = scale (q_lat . c_hat_t + q_pe' . k_rot_t)           (S = Q C^T)
//   o_lat = sum_t softmax(s)_t c_hat_t                           (O^T = C^T P^T)
//   out   = W_UV_h o_lat                                         (unabsorb)
// The attention is split over rows: the concatenation of all sequences'
// cache rows is cut into one equal range per CTA (persistent grid); each
// (range, sequence) piece is a segment whose unnormalized partial (o, max,
// sum) goes to its own slot, b + cta, and `combine` merges the slots of a
// sequence by their log-sum-exp.
//
// Tensor-core mapping, 64-row cache tiles (64 x 576 bf16 = 72 KB, 2 stages):
//   S[h, t]   : M = 64 heads, N = 64 rows, K = 576; A = q (resident), B = tile
//               (K-major), fp32 in TMEM lanes (h % 16) + 32 (h / 16).
//   O^T[d, h] : M = 128 latent dims (4 blocks), N = 64 heads, K = 64 rows;
//               A = the same tile read MN-major, B = P (K-major, from smem).
#pragma once
#include "tc_gemm.cuh"

namespace mla {
namespace tc {

constexpr int kDecRows = 64;                    // cache rows per tile
constexpr int kDecHeads = 64;                   // heads per CTA (M of S)
constexpr int kDecBoxes = 9;                    // 576 columns = 9 x 64
constexpr int kDecBoxBytes = kDecRows * 128;    // [64 rows x 64 cols] bf16
constexpr int kDecTileBytes = kDecBoxes * kDecBoxBytes;
constexpr int kDecQBytes = kDecBoxes * kDecHeads * 128;
constexpr int kDecPBytes = kDecHeads * 128;
constexpr int kDecThreads = 192;
constexpr size_t kDecSmem = (size_t)kDecQBytes + 2 * (size_t)kDecTileBytes + kDecPBytes + 1024;
constexpr int kDecOCol = 0;                     // O^T: 4 blocks x 64 columns
constexpr int kDecSCol = 256;                   // S: 64 columns (M = 64 layout)

// ---- split schedule -----------------------------------------------------------
// prefix[b] = rows of sequences before b (invalid sequences count 0 rows);
// prefix[B] = total; meta[0] = rows per CTA (ceil(total / G)).
__global__ void __launch_bounds__(1024)
decode_schedule_kernel(const int32_t* __restrict__ lens, const int64_t* __restrict__ offsets, int B, int max_len,
                       int64_t cache_rows, int G, int64_t* __restrict__ prefix, int64_t* __restrict__ meta) {
  __shared__ int64_t s_scan[1024];
  __shared__ int64_t s_carry;
  const int tid = threadIdx.x;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base <= B; base += blockDim.x) {
    const int b = base + tid;
    int64_t n = 0;
    if (b < B) {
      const int64_t L = lens[b], off = offsets[b];
      if (L < 1 || L > max_len || off < 0 || off + L > cache_rows) raise_device_error(kDevErrBadInput);
      else n = L;
    }
    s_scan[tid] = n;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
      const int64_t v = tid >= o ? s_scan[tid - o] : 0;
      __syncthreads();
      s_scan[tid] += v;
      __syncthreads();
    }
    if (b <= B) prefix[b] = s_carry + s_scan[tid] - n;
    __syncthreads();
    if (tid == (int)blockDim.x - 1) s_carry += s_scan[tid];
    __syncthreads();
  }
  if (tid == 0) {
    const int64_t total = s_carry;
    meta[0] = (total + G - 1) / G;
    meta[1] = total;
  }
}

// ---- q absorption and rotation (CUDA cores) --------------------------------------
// grid (H, R / 128 + 1). Blocks y < R/128: q_lat[b, h, 128 y .. +128] for every b
// with W_UK_h's column block resident in smem. Block y = R/128: q_pe rotated.
// Output qf [B, H, R + P] bf16 (the MMA operand dtype of the cache).
__global__ void __launch_bounds__(256)
decode_qprep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ W,
                    const int32_t* __restrict__ positions, const float* __restrict__ cos_t,
                    const float* __restrict__ sin_t, int max_pos, int B, int H, int R, int N, int P, int V,
                    int interleaved, __nv_bfloat16* __restrict__ qf) {
  extern __shared__ float s_w[];             // [N][128]
  __shared__ float s_q[2][512];
  const int h = blockIdx.x, yb = blockIdx.y;
  const int D = N + P, C = R + P;
  const int tid = threadIdx.x;
  if (yb * 128 < R) {
    const __nv_bfloat16* Wk = W + (int64_t)h * (N + V) * R + yb * 128;   // rows j < N of head h
    for (int e = tid; e < N * 128; e += 256) s_w[e] = __bfloat162float(Wk[(int64_t)(e / 128) * R + (e % 128)]);
    const int d = tid & 127, half = tid >> 7;
    for (int b0 = 0; b0 < B; b0 += 2) {
      __syncthreads();
      for (int e = tid; e < 2 * N; e += 256) {
        const int bb = b0 + e / N;
        s_q[e / N][e % N] = bb < B ? __bfloat162float(q[((int64_t)bb * H + h) * D + (e % N)]) : 0.f;
      }
      __syncthreads();
      const int b = b0 + half;
      if (b < B) {
        float a = 0.f;
        for (int j = 0; j < N; ++j) a = fmaf(s_w[j * 128 + d], s_q[half][j], a);
        qf[((int64_t)b * H + h) * C + yb * 128 + d] = __float2bfloat16_rn(a);
      }
    }
  } else {
    const int pairs = P / 2;
    for (int e = tid; e < B * pairs; e += 256) {
      const int b = e / pairs, i = e % pairs;
      int ia, ib;
      rope_pair_slots(i, P, interleaved, ia, ib);
      const int64_t pos = checked_pos(positions[b], max_pos);
      const __nv_bfloat16* qr = q + ((int64_t)b * H + h) * D + N;
      float ox, oy;
      rope_turn(__bfloat162float(qr[ia]), __bfloat162float(qr[ib]), cos_t[pos * pairs + i],
                sin_t[pos * pairs + i], ox, oy);
      __nv_bfloat16* dst = qf + ((int64_t)b * H + h) * C + R;
      dst[ia] = __float2bfloat16_rn(ox);
      dst[ib] = __float2bfloat16_rn(oy);
    }
  }
}

// ---- segments of one CTA's row range --------------------------------------------
struct DecSeg {
  int b;
  int64_t lo, hi;   // rows within sequence b
};
// Walks the pieces of [lo, hi) (concatenated row space) that fall in each
// sequence; returns false when done.
struct DecSegIter {
  const int64_t* prefix;
  int B;
  int64_t cur, end;
  int b;
  __device__ void init(const int64_t* pre, int nb, int64_t lo, int64_t hi) {
    prefix = pre; B = nb; cur = lo; end = hi;
    int l = 0, r = nb;                 // largest b with prefix[b] <= lo
    while (r - l > 1) { const int m = (l + r) >> 1; if (pre[m] <= lo) l = m; else r = m; }
    b = l;
  }
  __device__ bool next(DecSeg& s) {
    while (cur < end && b < B) {
      const int64_t p0 = prefix[b], p1 = prefix[b + 1];
      if (p1 > cur) {
        const int64_t e = p1 < end ? p1 : end;
        s.b = b; s.lo = cur - p0; s.hi = e - p0;
        cur = e;
        ++b;
        return true;
      }
      ++b;
    }
    return false;
  }
};

struct DecParams {
  const int64_t* prefix;
  const int64_t* meta;
  const int64_t* offsets;
  float* o_part;     // [slots, H, R]
  float* m_part;     // [slots, H] (log2 units)
  float* l_part;     // [slots, H]
  int B, H, R;
  float scale_log2;
};

struct DecBarriers {
  uint64_t q_full, q_empty;
  uint64_t c_full[2], c_empty[2];
  uint64_t s_full, s_free, p_full, pv_done, o_free, mma_done;
  uint64_t alpha_ready;   // the 128 softmax threads' per-tile exchange (bounded)
  uint32_t tmem_base;
  int abort_flag;
  float alpha[2][kDecHeads];
  int need[2][4];
};

__global__ void __launch_bounds__(kDecThreads, 1)
decode_attn_kernel(const __grid_constant__ CUtensorMap map_cache, const __grid_constant__ CUtensorMap map_q,
                   DecParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ DecBarriers bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x;
  const int64_t per = p.meta[0], total = p.meta[1];
  const int64_t r_lo = (int64_t)c * per;
  const int64_t r_hi = min(total, r_lo + per);
  if (r_lo >= r_hi) return;   // uniform over the CTA
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sC = smem + kDecQBytes;
  uint8_t* sP = sC + 2 * kDecTileBytes;
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < 2; ++s) { mbar_init(&bars.c_full[s], 1); mbar_init(&bars.c_empty[s], 1); }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.s_free, 128);
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.o_free, 128);
    mbar_init(&bars.mma_done, 1);
    mbar_init(&bars.alpha_ready, 128);
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
      tma_prefetch_desc(&map_cache);
      tma_prefetch_desc(&map_q);
      DecSegIter itr;
      itr.init(p.prefix, p.B, r_lo, r_hi);
      DecSeg sg;
      int it = 0, segi = 0;
      bool ok = true;
      while (ok && itr.next(sg)) {
        if (!mbar_wait(&bars.q_empty, ((uint32_t)segi & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars.q_full, kDecQBytes);
        for (int a = 0; a < kDecBoxes; ++a)
          tma_load_2d(sQ + a * kDecHeads * 128, &map_q, &bars.q_full, a * 64, sg.b * kDecHeads);
        const int64_t row0 = p.offsets[sg.b] + sg.lo;
        const int ntiles = (int)((sg.hi - sg.lo + kDecRows - 1) / kDecRows);
        for (int k = 0; k < ntiles; ++k, ++it) {
          const int s = it & 1;
          if (!mbar_wait(&bars.c_empty[s], ((uint32_t)(it >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.c_full[s], kDecTileBytes);
          uint8_t* st = sC + s * kDecTileBytes;
          for (int a = 0; a < kDecBoxes; ++a)
            tma_load_2d(st + a * kDecBoxBytes, &map_cache, &bars.c_full[s], a * 64, (int)(row0 + (int64_t)k * kDecRows));
        }
        ++segi;
      }
      if (!ok) {   // let the copies in flight land before the CTA exits
        if (segi > 0 || it > 0) mbar_wait_drain(&bars.q_full, (uint32_t)(segi > 0 ? segi - 1 : 0) & 1u);
        for (int i = (it > 2 ? it - 2 : 0); i < it; ++i) mbar_wait_drain(&bars.c_full[i & 1], (uint32_t)(i >> 1) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kDecHeads, kDecRows);
      const uint32_t idesc_o = idesc_bf16_f32(128, kDecHeads) | kIdescAMajorMN;
      const uint32_t s_tmem = tmem + kDecSCol;
      // The (segment, tile) items form one stream; S of item i+1 is issued
      // before P V of item i, so the next scores overlap this tile's softmax.
      struct Item { int seg; bool first, last; };
      DecSegIter itr;
      itr.init(p.prefix, p.B, r_lo, r_hi);
      DecSeg cur;
      bool have = itr.next(cur);
      int segi = 0, k_in_seg = 0;
      int nt = have ? (int)((cur.hi - cur.lo + kDecRows - 1) / kDecRows) : 0;
      auto next_item = [&](Item& out) -> bool {
        if (!have) return false;
        out.seg = segi;
        out.first = (k_in_seg == 0);
        out.last = (k_in_seg == nt - 1);
        if (++k_in_seg == nt) {
          ++segi;
          k_in_seg = 0;
          have = itr.next(cur);
          nt = have ? (int)((cur.hi - cur.lo + kDecRows - 1) / kDecRows) : 0;
        }
        return true;
      };
      auto issue_s = [&](int item, const Item& itm) -> bool {
        const int s = item & 1;
        if (itm.first && !mbar_wait(&bars.q_full, (uint32_t)itm.seg & 1u, abort_flag)) return false;
        if (!mbar_wait(&bars.c_full[s], (uint32_t)(item >> 1) & 1u, abort_flag)) return false;
        if (!mbar_wait(&bars.s_free, ((uint32_t)item & 1u) ^ 1u, abort_flag)) return false;
        tc_fence_after();
        const uint8_t* st = sC + s * kDecTileBytes;
#pragma unroll 1
        for (int a = 0; a < kDecBoxes; ++a) {
          const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + a * kDecHeads * 128));
          const uint64_t cd = desc_kmajor_sw128(smem_u32(st + a * kDecBoxBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ss(s_tmem, desc_advance(qd, k * 32), desc_advance(cd, k * 32), idesc_s, (a | k) != 0);
        }
        mma_commit(&bars.s_full);
        if (itm.last) mma_commit(&bars.q_empty);   // q may be replaced once these are done
        return true;
      };
      auto issue_pv = [&](int item, const Item& itm) -> bool {
        const int s = item & 1;
        if (itm.first && itm.seg > 0 && !mbar_wait(&bars.o_free, (uint32_t)(itm.seg - 1) & 1u, abort_flag))
          return false;
        if (!mbar_wait(&bars.p_full, (uint32_t)item & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint8_t* st = sC + s * kDecTileBytes;
        const uint64_t pd = desc_kmajor_sw128(smem_u32(sP));
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
          // latent columns [128 blk, 128 blk + 128) = boxes 2 blk, 2 blk + 1, read MN-major
          const uint64_t ad = desc_mnmajor_sw128(smem_u32(st + 2 * blk * kDecBoxBytes), kDecBoxBytes, 1024);
#pragma unroll
          for (int k = 0; k < kDecRows / 16; ++k)
            mma_bf16_ss(tmem + kDecOCol + blk * kDecHeads, desc_advance(ad, k * 2048), desc_advance(pd, k * 32),
                        idesc_o, (itm.first && k == 0) ? 0u : 1u);
        }
        mma_commit(&bars.c_empty[s]);
        mma_commit(&bars.pv_done);
        return true;
      };
      Item a_item;
      int item = 0;
      if (next_item(a_item) && issue_s(0, a_item)) {
        for (;;) {
          Item b_item;
          const bool has_next = next_item(b_item);
          if (has_next && !issue_s(item + 1, b_item)) break;
          if (!issue_pv(item, a_item)) break;
          if (!has_next) break;
          a_item = b_item;
          ++item;
        }
      }
      mma_commit(&bars.mma_done);          // every MMA done before TMEM is freed
      mbar_wait_drain(&bars.mma_done, 0);
    }
  } else {
    // ---------------- softmax / correction / partial epilogue (warps 2-5) ----------------
    const int grp = warp & 3;                       // TMEM quadrant
    const bool owner = lane < 16;                   // S row owner (M = 64 layout)
    const int h = grp * 16 + (lane & 15);           // head of this S row (owners)
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    const int d_lane = grp * 32 + lane;             // O^T row (latent dim within a block)
    DecSegIter itr;
    itr.init(p.prefix, p.B, r_lo, r_hi);
    DecSeg sg;
    int it = 0, segi = 0;
    bool ok = true;
    while (ok && itr.next(sg)) {
      const int slot = sg.b + c;
      const int ntiles = (int)((sg.hi - sg.lo + kDecRows - 1) / kDecRows);
      float m = -INFINITY, l = 0.f;
      for (int k = 0; k < ntiles; ++k, ++it) {
        const int par = it & 1;
        if (!mbar_wait_warp(&bars.s_full, (uint32_t)it & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float sc[kDecRows];
#pragma unroll
        for (int cc = 0; cc < kDecRows / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + (uint32_t)(kDecSCol + cc * 16), v);
#pragma unroll
          for (int e = 0; e < 16; ++e) sc[cc * 16 + e] = __uint_as_float(v[e]);
        }
        tc_fence_before();
        mbar_arrive(&bars.s_free);
        const int64_t t0 = sg.lo + (int64_t)k * kDecRows;
        const int nvalid = (int)min((int64_t)kDecRows, sg.hi - t0);
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < kDecRows; ++e) {
          const float x = (e < nvalid) ? sc[e] * p.scale_log2 : -INFINITY;
          sc[e] = x;
          mx = fmaxf(mx, x);
        }
        // reference max: raised only when a row's max grows by more than 8
        // (P then stays below 2^8), so O is rarely rescaled
        float alpha = 1.f;
        bool need = false;
        if (owner && mx > m + 8.f) {
          alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - mx);
          need = (k > 0);
          m = mx;
        }
        uint32_t pk[kDecRows / 2];
        float rs = 0.f;
#pragma unroll
        for (int e = 0; e < kDecRows; e += 2) {
          pk[e / 2] = pack_bf16x2(ex2_approx(sc[e] - m), ex2_approx(sc[e + 1] - m));
          const float2 pr = unpack_bf16x2(pk[e / 2]);
          rs += pr.x + pr.y;
        }
        l = l * alpha + rs;
        if (owner) bars.alpha[par][h] = alpha;
        const bool wneed = __any_sync(0xffffffffu, need);
        if (lane == 0) bars.need[par][grp] = wneed ? 1 : 0;
        // previous P V done: P buffer free and O stable
        if (it > 0 && !mbar_wait_warp(&bars.pv_done, (uint32_t)(it - 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        mbar_arrive(&bars.alpha_ready);   // alpha / need of this tile published
        if (!mbar_wait_warp(&bars.alpha_ready, (uint32_t)it & 1u, abort_flag)) { ok = false; break; }
        const bool any_need = (bars.need[par][0] | bars.need[par][1] | bars.need[par][2] | bars.need[par][3]) != 0;
        if (any_need) {
          // O^T[d, h] *= alpha[h]: this thread owns TMEM lane d of every block
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk)
#pragma unroll 1
            for (int cc = 0; cc < kDecHeads / 16; ++cc) {
              uint32_t v[16];
              const uint32_t ta = tmem + lane_base + (uint32_t)(kDecOCol + blk * kDecHeads + cc * 16);
              tmem_ld16(ta, v);
#pragma unroll
              for (int e = 0; e < 16; ++e)
                v[e] = __float_as_uint(__uint_as_float(v[e]) * bars.alpha[par][cc * 16 + e]);
              tmem_st16(ta, v);
            }
          tmem_st_wait();
        }
        if (owner) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            *reinterpret_cast<uint4*>(sP + sw128_offset(h, cc)) =
                make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars.p_full);
      }
      if (!ok) break;
      // segment epilogue: unnormalized partial to slot (b + cta)
      if (!mbar_wait_warp(&bars.pv_done, (uint32_t)(it - 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float* op = p.o_part + (int64_t)slot * p.H * p.R;
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk)
#pragma unroll 1
        for (int cc = 0; cc < kDecHeads / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + (uint32_t)(kDecOCol + blk * kDecHeads + cc * 16), v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            op[(int64_t)(cc * 16 + e) * p.R + blk * 128 + d_lane] = __uint_as_float(v[e]);
        }
      if (owner) {
        p.m_part[(int64_t)slot * p.H + h] = m;
        p.l_part[(int64_t)slot * p.H + h] = l;
      }
      tc_fence_before();
      mbar_arrive(&bars.o_free);
      ++segi;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- merge the partials of each (b, h) ----------------------------------------
// o_lat[b, h, :] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the slots
// b + c of the CTAs c whose ranges touch sequence b.
__global__ void __launch_bounds__(128)
decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ m_part,
                      const float* __restrict__ l_part, const int64_t* __restrict__ prefix,
                      const int64_t* __restrict__ meta, int H, int R, float* __restrict__ o_lat) {
  const int b = blockIdx.x, h = blockIdx.y;
  const int64_t per = meta[0];
  const int64_t p0 = prefix[b], p1 = prefix[b + 1];
  float* dst = o_lat + ((int64_t)b * H + h) * R;
  if (p1 <= p0 || per <= 0) {   // a skipped sequence: no row to attend
    for (int d = threadIdx.x; d < R; d += blockDim.x) dst[d] = 0.f;
    return;
  }
  const int c0 = (int)(p0 / per), c1 = (int)((p1 - 1) / per);
  float M = -INFINITY;
  for (int cc = c0; cc <= c1; ++cc) M = fmaxf(M, m_part[(int64_t)(b + cc) * H + h]);
  float Lsum = 0.f;
  for (int cc = c0; cc <= c1; ++cc) {
    const float ms = m_part[(int64_t)(b + cc) * H + h];
    Lsum += (ms == -INFINITY ? 0.f : exp2f(ms - M)) * l_part[(int64_t)(b + cc) * H + h];
  }
  const float inv = 1.f / Lsum;
  for (int d = threadIdx.x; d < R; d += blockDim.x) {
    float a = 0.f;
    for (int cc = c0; cc <= c1; ++cc) {
      const int64_t slot = b + cc;
      const float ms = m_part[slot * H + h];
      if (ms != -INFINITY) a = fmaf(exp2f(ms - M), o_part[(slot * H + h) * R + d], a);
    }
    dst[d] = a * inv;
  }
}

// ---- out[b, h, :] = W_UV_h o_lat[b, h, :] ----------------------------------------
// grid (H, V / 32): W_UV_h's 32-row block resident in smem, looped over b.
__global__ void __launch_bounds__(256)
decode_unabsorb_kernel(const float* __restrict__ o_lat, const __nv_bfloat16* __restrict__ W, int B, int H, int R,
                       int N, int V, __nv_bfloat16* __restrict__ out) {
  extern __shared__ float s_wv[];            // [32][R]
  __shared__ float s_o[512];
  const int h = blockIdx.x, c0 = blockIdx.y * 32;
  const int nc = min(32, V - c0);
  const __nv_bfloat16* Wv = W + ((int64_t)h * (N + V) + N + c0) * R;
  for (int e = threadIdx.x; e < nc * R; e += blockDim.x) s_wv[e] = __bfloat162float(Wv[e]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int b = 0; b < B; ++b) {
    __syncthreads();
    for (int d = threadIdx.x; d < R; d += blockDim.x) s_o[d] = o_lat[((int64_t)b * H + h) * R + d];
    __syncthreads();
    for (int cc = warp; cc < nc; cc += 8) {
      float a = 0.f;
      for (int d = lane; d < R; d += 32) a = fmaf(s_wv[cc * R + d], s_o[d], a);
      a = warp_sum(a);
      if (lane == 0) out[((int64_t)b * H + h) * V + c0 + cc] = __float2bfloat16_rn(a);
    }
  }
}

}  // namespace tc
}  // namespace mla
