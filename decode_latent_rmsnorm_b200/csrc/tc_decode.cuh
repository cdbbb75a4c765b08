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
// Tensor-core mapping, 32-row cache tiles (32 x 576 bf16 = 36 KB) in a
// 4-stage TMA ring, so three tiles are in flight while one is computed:
//   S[h, t] : M = 64 heads, N = 32 rows, K = 576; A = q (resident), B = tile
//             (K-major); fp32 in TMEM lanes (h % 16) + 32 (h / 16).
//   O[h, d] : M = 64 heads, N = 256 latent dims (two accumulators, lower and
//             upper 16 lanes of each quadrant), K = 32 rows; A = P (smem),
//             B = the same cache tile read MN-major.
#pragma once
#include "tc_gemm.cuh"

namespace mla {
namespace tc {

constexpr int kDecRows = 32;                    // cache rows per tile
constexpr int kDecStages = 4;                   // TMA ring depth
constexpr int kDecHeads = 64;                   // heads per CTA (M of S)
constexpr int kDecBoxes = 9;                    // 576 columns = 9 x 64
constexpr int kDecBoxBytes = kDecRows * 128;    // [32 rows x 64 cols] bf16
constexpr int kDecTileBytes = kDecBoxes * kDecBoxBytes;
constexpr int kDecQBytes = kDecBoxes * kDecHeads * 128;
constexpr int kDecPBytes = 2 * kDecHeads * kDecRows * 2;   // two [64 heads x 32 rows] bf16
constexpr int kDecThreads = 192;
constexpr size_t kDecSmem = (size_t)kDecQBytes + kDecStages * (size_t)kDecTileBytes + kDecPBytes + 1024;
constexpr int kDecOCol = 0;                     // O: 256 columns (both lane halves)
constexpr int kDecSCol = 256;                   // S: 2 x 32 columns (M = 64 layout)

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

// ---- per-head batched GEMM on CUDA cores (q absorption, un-absorption) ----------
// For head h (grid x) and a 64-column block (grid y) and 64-row block (grid z):
//   C[m, n] = sum_k A[m, k] * Bm[k, n]   (fp32 accumulate, bf16 output)
// with A[m, k] = a[m * a_ms + h * a_hs + k] and
//   b_kn = true : Bm[k, n] = w[h * w_hs + k * w_ks + n]   (rows k, n contiguous)
//   b_kn = false: Bm[k, n] = w[h * w_hs + n * w_ks + k]   (rows n, k contiguous)
// C[m, n] goes to c[m * c_ms + h * c_hs + n]. 256 threads, 4 x 4 outputs per
// thread, K in chunks of 32 staged in smem ([k][m], [k][n], fp32).
constexpr int kSgBM = 64, kSgBN = 64, kSgBK = 32, kSgPad = 68;
template <typename TA, bool kBKN>
__global__ void __launch_bounds__(256)
small_gemm_kernel(const TA* __restrict__ a, int64_t a_ms, int64_t a_hs, const __nv_bfloat16* __restrict__ w,
                  int64_t w_hs, int64_t w_ks, __nv_bfloat16* __restrict__ cout, int64_t c_ms, int64_t c_hs,
                  int M, int N, int K) {
  __shared__ __align__(16) float sA[kSgBK][kSgPad];
  __shared__ __align__(16) float sB[kSgBK][kSgPad];
  const int h = blockIdx.x, n0 = blockIdx.y * kSgBN, m0 = blockIdx.z * kSgBM;
  const int tid = threadIdx.x;
  const int tm = (tid >> 4) * 4, tn = (tid & 15) * 4;
  float acc[4][4] = {};
  const TA* ah = a + (int64_t)h * a_hs;
  const __nv_bfloat16* wh = w + (int64_t)h * w_hs;
  for (int k0 = 0; k0 < K; k0 += kSgBK) {
    __syncthreads();
    for (int e = tid; e < kSgBM * kSgBK; e += 256) {          // A chunk, k fastest (coalesced)
      const int mm = e / kSgBK, kk = e % kSgBK;
      const int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < M && k < K) v = to_f32(ah[(int64_t)m * a_ms + k]);
      sA[kk][mm] = v;
    }
    for (int e = tid; e < kSgBN * kSgBK; e += 256) {
      int nn, kk;
      if (kBKN) { kk = e / kSgBN; nn = e % kSgBN; } else { nn = e / kSgBK; kk = e % kSgBK; }
      const int n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < N && k < K) v = __bfloat162float(kBKN ? wh[(int64_t)k * w_ks + n] : wh[(int64_t)n * w_ks + k]);
      sB[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kSgBK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(&sA[kk][tm]);
      const float4 bv = *reinterpret_cast<const float4*>(&sB[kk][tn]);
      const float ar[4] = {av.x, av.y, av.z, av.w}, br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jx = 0; jx < 4; ++jx) acc[i][jx] = fmaf(ar[i], br[jx], acc[i][jx]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm + i;
    if (m >= M) continue;
    __nv_bfloat16* dst = cout + (int64_t)m * c_ms + (int64_t)h * c_hs + n0 + tn;
    if (n0 + tn + 3 < N) {
      uint2 v2 = make_uint2(pack_bf16x2(acc[i][0], acc[i][1]), pack_bf16x2(acc[i][2], acc[i][3]));
      *reinterpret_cast<uint2*>(dst) = v2;
    } else {
#pragma unroll
      for (int jx = 0; jx < 4; ++jx)
        if (n0 + tn + jx < N) dst[jx] = __float2bfloat16_rn(acc[i][jx]);
    }
  }
}

// q_pe rotated at the query position, into the last P columns of qf rows.
__global__ void decode_qrope_kernel(const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ positions,
                                    const float* __restrict__ cos_t, const float* __restrict__ sin_t, int max_pos,
                                    int B, int H, int R, int N, int P, int interleaved,
                                    __nv_bfloat16* __restrict__ qf) {
  const int pairs = P / 2;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)B * H * pairs) return;
  const int i = (int)(e % pairs);
  const int64_t bh = e / pairs;
  const int b = (int)(bh / H);
  int ia, ib;
  rope_pair_slots(i, P, interleaved, ia, ib);
  const int64_t pos = checked_pos(positions[b], max_pos);
  const __nv_bfloat16* qr = q + bh * (N + P) + N;
  float ox, oy;
  rope_turn(__bfloat162float(qr[ia]), __bfloat162float(qr[ib]), cos_t[pos * pairs + i], sin_t[pos * pairs + i], ox,
            oy);
  __nv_bfloat16* dst = qf + bh * (R + P) + R;
  dst[ia] = __float2bfloat16_rn(ox);
  dst[ib] = __float2bfloat16_rn(oy);
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
  uint64_t c_full[kDecStages], c_empty[kDecStages];
  uint64_t s_full[2], s_free[2];     // S double buffer (TMEM)
  uint64_t p_full[2], pv_done[2];    // P double buffer (smem)
  uint64_t o_free, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// One persistent CTA per SM; warp 0 issues TMA loads, warp 1 the MMAs, warps
// 2-5 run the softmax. TMEM (512 columns):
//   O[h, d]  (M = 64 accumulators): d < 256 in the lower 16 lanes of each
//            32-lane quadrant, d >= 256 in the upper 16 lanes, columns 0-255;
//   S[h, t]  two 32-column buffers at columns 256 and 288, lower lanes.
// Head h = 16 q + i (quadrant q, lane i < 16) is owned by lanes i and i + 16
// of warp q: the lower lane runs h's online softmax, both rescale their half
// of h's O row, so the softmax needs no exchange across warps.
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
  uint8_t* sP = sC + kDecStages * kDecTileBytes;            // 2 x [64 heads x 32 rows], no swizzle
  constexpr int kPBuf = kDecHeads * kDecRows * 2;           // 4 KB
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int s = 0; s < kDecStages; ++s) { mbar_init(&bars.c_full[s], 1); mbar_init(&bars.c_empty[s], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.s_full[b], 1);
      mbar_init(&bars.s_free[b], 128);
      mbar_init(&bars.p_full[b], 128);
      mbar_init(&bars.pv_done[b], 1);
    }
    mbar_init(&bars.o_free, 128);
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
          const int s = it % kDecStages;
          if (!mbar_wait(&bars.c_empty[s], ((uint32_t)(it / kDecStages) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.c_full[s], kDecTileBytes);
          uint8_t* st = sC + s * kDecTileBytes;
          for (int a = 0; a < kDecBoxes; ++a)
            tma_load_2d(st + a * kDecBoxBytes, &map_cache, &bars.c_full[s], a * 64,
                        (int)(row0 + (int64_t)k * kDecRows));
        }
        ++segi;
      }
      if (!ok) {   // let the copies in flight land before the CTA exits
        if (segi > 0) mbar_wait_drain(&bars.q_full, (uint32_t)(segi - 1) & 1u);
        for (int i = (it > kDecStages ? it - kDecStages : 0); i < it; ++i)
          mbar_wait_drain(&bars.c_full[i % kDecStages], (uint32_t)(i / kDecStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kDecHeads, kDecRows);
      const uint32_t idesc_o = idesc_bf16_f32(kDecHeads, 256) | kIdescBMajorMN;
      // The (segment, tile) items form one stream. S runs two items ahead of
      // P V: S(j + 2) is issued right after P V(j).
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
      auto issue_s = [&](int j, const Item& itm) -> bool {
        const int s = j % kDecStages, b = j & 1;
        if (itm.first && !mbar_wait(&bars.q_full, (uint32_t)itm.seg & 1u, abort_flag)) return false;
        if (!mbar_wait(&bars.c_full[s], (uint32_t)(j / kDecStages) & 1u, abort_flag)) return false;
        if (!mbar_wait(&bars.s_free[b], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) return false;
        tc_fence_after();
        const uint8_t* st = sC + s * kDecTileBytes;
        const uint32_t s_tmem = tmem + kDecSCol + b * kDecRows;
#pragma unroll 1
        for (int a = 0; a < kDecBoxes; ++a) {
          const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + a * kDecHeads * 128));
          const uint64_t cd = desc_kmajor_sw128(smem_u32(st + a * kDecBoxBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ss(s_tmem, desc_advance(qd, k * 32), desc_advance(cd, k * 32), idesc_s, (a | k) != 0);
        }
        mma_commit(&bars.s_full[b]);
        if (itm.last) mma_commit(&bars.q_empty);   // q may be replaced once these are done
        return true;
      };
      auto issue_pv = [&](int j, const Item& itm) -> bool {
        const int s = j % kDecStages, b = j & 1;
        if (itm.first && itm.seg > 0 && !mbar_wait(&bars.o_free, (uint32_t)(itm.seg - 1) & 1u, abort_flag))
          return false;
        if (!mbar_wait(&bars.p_full[b], (uint32_t)(j >> 1) & 1u, abort_flag)) return false;
        tc_fence_after();
        const uint8_t* st = sC + s * kDecTileBytes;
        const uint64_t pd = desc_kmajor_noswz(smem_u32(sP + b * kPBuf), 128, 512);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          // latent columns [256 half, 256 half + 256) = boxes 4 half .. 4 half + 3, read MN-major
          const uint64_t cd = desc_mnmajor_sw128(smem_u32(st + 4 * half * kDecBoxBytes), kDecBoxBytes, 1024);
          const uint32_t o_tmem = tmem + kDecOCol + ((uint32_t)(16 * half) << 16);
#pragma unroll
          for (int k = 0; k < kDecRows / 16; ++k)
            mma_bf16_ss(o_tmem, desc_advance(pd, k * 256), desc_advance(cd, k * 2048), idesc_o,
                        (itm.first && k == 0) ? 0u : 1u);
        }
        mma_commit(&bars.c_empty[s]);
        mma_commit(&bars.pv_done[b]);
        return true;
      };
      Item win[3];   // items j, j+1, j+2
      int nwin = 0;
      for (; nwin < 2 && next_item(win[nwin]); ++nwin) {}
      bool ok = true;
      for (int i = 0; i < nwin && ok; ++i) ok = issue_s(i, win[i]);
      int j = 0;
      while (ok && nwin > 0) {
        if (!issue_pv(j, win[0])) break;
        Item nx;
        const bool more = next_item(nx);
        win[0] = win[1];
        if (more) {
          win[1] = nx;
          if (!issue_s(j + 2, nx)) break;
        } else {
          --nwin;
        }
        ++j;
        if (nwin == 1 && !more) {
          // one item left (j): its S is issued; finish with its P V
          if (!issue_pv(j, win[0])) break;
          break;
        }
      }
      mma_commit(&bars.mma_done);          // every MMA done before TMEM is freed
      mbar_wait_drain(&bars.mma_done, 0);
    }
  } else {
    // ---------------- softmax / correction / partial epilogue (warps 2-5) ----------------
    const int grp = warp & 3;                       // TMEM quadrant
    const bool lower = lane < 16;                   // S row owner (M = 64 layout)
    const int h = grp * 16 + (lane & 15);           // head of this lane pair
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    DecSegIter itr;
    itr.init(p.prefix, p.B, r_lo, r_hi);
    DecSeg sg;
    int j = 0, segi = 0;
    bool ok = true;
    while (ok && itr.next(sg)) {
      const int slot = sg.b + c;
      const int ntiles = (int)((sg.hi - sg.lo + kDecRows - 1) / kDecRows);
      float m = -INFINITY, l = 0.f;
      for (int k = 0; k < ntiles; ++k, ++j) {
        const int b = j & 1;
        if (!mbar_wait_warp(&bars.s_full[b], (uint32_t)(j >> 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float sc[kDecRows];
#pragma unroll
        for (int cc = 0; cc < kDecRows / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + (uint32_t)(kDecSCol + b * kDecRows + cc * 16), v);
#pragma unroll
          for (int e = 0; e < 16; ++e) sc[cc * 16 + e] = __uint_as_float(v[e]);
        }
        tc_fence_before();
        mbar_arrive(&bars.s_free[b]);
        const int64_t t0 = sg.lo + (int64_t)k * kDecRows;
        const int nvalid = (int)min((int64_t)kDecRows, sg.hi - t0);
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < kDecRows; ++e) {
          const float x = (e < nvalid) ? sc[e] * p.scale_log2 : -INFINITY;
          sc[e] = x;
          mx = fmaxf(mx, x);
        }
        // reference max: raised only when the row max grows by more than 8
        // (P then stays below 2^8), so O is rarely rescaled
        float alpha = 1.f;
        bool need = false;
        if (lower && mx > m + 8.f) {
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
        // both lanes of a head take the lower lane's alpha
        const float alpha_h = __shfl_sync(0xffffffffu, alpha, lane & 15);
        if (__any_sync(0xffffffffu, need)) {
          // O must be stable: the previous tile's P V is done
          if (k > 0 && !mbar_wait_warp(&bars.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 256 / 16; ++cc) {
            uint32_t v[16];
            const uint32_t ta = tmem + lane_base + (uint32_t)(kDecOCol + cc * 16);
            tmem_ld16(ta, v);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha_h);
            tmem_st16(ta, v);
          }
          tmem_st_wait();
        }
        // P buffer b is free once P V of tile j - 2 is done
        if (j >= 2 && !mbar_wait_warp(&bars.pv_done[b], (uint32_t)((j - 2) >> 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (lower) {
          // no-swizzle K-major layout: core matrix (h / 8, chunk) at (h / 8) * 512 + chunk * 128
          uint8_t* prow = sP + b * kPBuf + (h >> 3) * 512 + (h & 7) * 16;
#pragma unroll
          for (int cc = 0; cc < kDecRows / 8; ++cc)
            *reinterpret_cast<uint4*>(prow + cc * 128) = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars.p_full[b]);
      }
      if (!ok) break;
      // segment epilogue: unnormalized partial to slot (b + cta)
      if (!mbar_wait_warp(&bars.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float* op = p.o_part + ((int64_t)slot * p.H + h) * p.R + (lower ? 0 : 256);
#pragma unroll 1
      for (int cc = 0; cc < 256 / 16; ++cc) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(kDecOCol + cc * 16), v);
        float4* o4 = reinterpret_cast<float4*>(op + cc * 16);
        o4[0] = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]), __uint_as_float(v[3]));
        o4[1] = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]), __uint_as_float(v[7]));
        o4[2] = make_float4(__uint_as_float(v[8]), __uint_as_float(v[9]), __uint_as_float(v[10]), __uint_as_float(v[11]));
        o4[3] = make_float4(__uint_as_float(v[12]), __uint_as_float(v[13]), __uint_as_float(v[14]), __uint_as_float(v[15]));
      }
      if (lower) {
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

}  // namespace tc
}  // namespace mla
