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
// Tensor-core mapping (see decode_attn_kernel for the data flow):
//   S^T[t, h] : M = 64 cache rows, N = 64 heads, K = 576.
//   O^T[d, h] : M = 128 latent dims (4 blocks), N = 64 heads, K = 64 rows.
#pragma once
#include "tc_gemm.cuh"

namespace mla {
namespace tc {

constexpr int kDecRows = 64;                    // cache rows per tile (M of the score MMAs)
constexpr int kDecHeads = 64;                   // heads per CTA (N of both MMAs)
constexpr int kDecBoxes = 9;                    // 576 columns = 9 x 64
constexpr int kDecLatBoxes = 8;                 // the 512 latent columns
constexpr int kDecBoxBytes = kDecRows * 128;    // [64 rows x 64 cols] bf16 = 8 KB
constexpr int kDecBufs = 2;                     // tile buffers: one fills while the other is in use
constexpr int kDecBufBytes = kDecBoxes * kDecBoxBytes;
constexpr int kDecQBytes = kDecBoxes * kDecHeads * 128;
constexpr int kDecThreads = 192;
constexpr size_t kDecSmem = (size_t)kDecQBytes + kDecBufs * (size_t)kDecBufBytes + 1024;   // P^T reuses a rope box
constexpr int kDecOCol = 0;                     // O^T: 4 blocks x 64 columns
constexpr int kDecSCol = 256;                   // S^T: two buffers of 64 columns

// ---- split schedule -----------------------------------------------------------
// prefix[b] = rows of sequences before b (invalid sequences count 0 rows);
// prefix[B] = total; meta[0] = rows per CTA (ceil(total / G)).
// Run by one whole block (any size up to 1024 threads).
__device__ __forceinline__ void decode_schedule_block(const int32_t* __restrict__ lens,
                                                      const int64_t* __restrict__ offsets, int B, int max_len,
                                                      int64_t cache_rows, int G, int64_t* __restrict__ prefix,
                                                      int64_t* __restrict__ meta) {
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

// q_pe rotated at the query position, into the last P columns of qf rows.
// q_pe of sequences [b0, b0 + nb) and head h (q holds H heads per sequence),
// rotated at each sequence's position, into qf[b, h, R:] (bf16; qf holds Hq
// heads per sequence). Rotary width P = 64: the 128 calling
// threads take one sequence and half of its 32 pairs each, as vector loads
// (half-split pairing: values [16 hp, 16 hp + 16) and [32 + 16 hp, 48 + 16 hp);
// interleaved: values [32 hp, 32 hp + 32)).
__device__ __forceinline__ void decode_qrope_rows(const __nv_bfloat16* __restrict__ q,
                                                  const int32_t* __restrict__ positions,
                                                  const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                                                  int max_pos, int h, int b0, int nb, int H, int Hq, int R,
                                                  int N, int interleaved, __nv_bfloat16* __restrict__ qf,
                                                  int tid) {
  const int b = b0 + (tid >> 1), hp = tid & 1;
  if ((tid >> 1) >= nb) return;
  const int64_t pos = checked_pos(positions[b], max_pos);
  const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t)b * H + h) * (N + 64) + N);
  uint4* dst = reinterpret_cast<uint4*>(qf + ((int64_t)b * Hq + h) * (R + 64) + R);
  const float4* c4 = reinterpret_cast<const float4*>(cos_t + pos * 32 + hp * 16);
  const float4* s4 = reinterpret_cast<const float4*>(sin_t + pos * 32 + hp * 16);
  int ch[4];   // 16-byte chunks (8 values) of the row holding this thread's pairs
  if (interleaved) {
    ch[0] = 4 * hp; ch[1] = 4 * hp + 1; ch[2] = 4 * hp + 2; ch[3] = 4 * hp + 3;
  } else {
    ch[0] = 2 * hp; ch[1] = 2 * hp + 1; ch[2] = 4 + 2 * hp; ch[3] = 5 + 2 * hp;
  }
  uint4 raw[4];
  float4 cv[4], sv[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) { raw[k] = src[ch[k]]; cv[k] = c4[k]; sv[k] = s4[k]; }
  float x[32], cs[16], sn[16];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t w4[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w4[e]);
      x[k * 8 + 2 * e] = f.x;
      x[k * 8 + 2 * e + 1] = f.y;
    }
    cs[4 * k] = cv[k].x; cs[4 * k + 1] = cv[k].y; cs[4 * k + 2] = cv[k].z; cs[4 * k + 3] = cv[k].w;
    sn[4 * k] = sv[k].x; sn[4 * k + 1] = sv[k].y; sn[4 * k + 2] = sv[k].z; sn[4 * k + 3] = sv[k].w;
  }
  // local pair i: (x[2i], x[2i+1]) when interleaved, (x[i], x[16+i]) otherwise
  float y[32];
  if (interleaved) {
#pragma unroll
    for (int i = 0; i < 16; ++i) rope_turn(x[2 * i], x[2 * i + 1], cs[i], sn[i], y[2 * i], y[2 * i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) rope_turn(x[i], x[16 + i], cs[i], sn[i], y[i], y[16 + i]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    dst[ch[k]] = make_uint4(pack_bf16x2(y[k * 8], y[k * 8 + 1]), pack_bf16x2(y[k * 8 + 2], y[k * 8 + 3]),
                            pack_bf16x2(y[k * 8 + 4], y[k * 8 + 5]), pack_bf16x2(y[k * 8 + 6], y[k * 8 + 7]));
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

// The (segment, tile) stream every role of a CTA walks in the same order.
struct DecTile {
  int seg, b;
  int64_t row0;      // first cache row of the tile
  int nvalid;        // rows of the tile inside the segment
  bool first, last;  // first / last tile of its segment
};
struct DecTileIter {
  DecSegIter segs;
  const int64_t* offsets;
  DecSeg cur;
  bool have;
  int segi, k, nt;
  __device__ void init(const DecParams& p, int64_t lo, int64_t hi) {
    segs.init(p.prefix, p.B, lo, hi);
    offsets = p.offsets;
    have = segs.next(cur);
    segi = 0;
    k = 0;
    nt = have ? (int)((cur.hi - cur.lo + kDecRows - 1) / kDecRows) : 0;
  }
  __device__ bool next(DecTile& t) {
    if (!have) return false;
    t.seg = segi;
    t.b = cur.b;
    const int64_t r = cur.lo + (int64_t)k * kDecRows;
    t.row0 = offsets[cur.b] + r;
    t.nvalid = (int)min((int64_t)kDecRows, cur.hi - r);
    t.first = (k == 0);
    t.last = (k == nt - 1);
    if (++k == nt) {
      ++segi;
      k = 0;
      have = segs.next(cur);
      nt = have ? (int)((cur.hi - cur.lo + kDecRows - 1) / kDecRows) : 0;
    }
    return true;
  }
};

struct DecBarriers {
  uint64_t q_full, q_empty;
  uint64_t full[kDecBufs], empty[kDecBufs];   // a tile buffer: its nine boxes landed / free again
  uint64_t s_full[2], s_free[2];              // S^T buffers (TMEM)
  uint64_t p_full[2];                         // P^T of the tile in buffer b (smem, its rope box)
  uint64_t pv_done[2], o_free, mma_done;   // pv_done[j & 1]: the latent product of tile j
  uint64_t sm_sync;                           // bounded barrier of the 128 softmax threads
  uint32_t tmem_base;
  int abort_flag;
  int vote[2][4];                    // per tile parity: a vote is read after one sync, rewritten after two
  alignas(16) float m_ref[kDecHeads];   // per-head reference max (log2 units; read as float4)
  float alpha[kDecHeads];
  float red[4][kDecHeads];           // per-warp column maxima / sums
};

// Column reduction over each half of a warp: lane l holds v[0..31], the
// values of heads 32 (l >> 4) + i of one row, and ends with the reduction
// over the 16 lanes of its half of heads 32 (l >> 4) + 2 (l & 15) and the
// one after (a halving exchange: 16 + 8 + 4 + 2 shuffles).
template <bool kMax>
__device__ __forceinline__ float2 half_column_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    const bool up = (lane & m) != 0;
#pragma unroll
    for (int c = 0; c < 2 * m; ++c) {
      const float send = up ? v[c] : v[c + 2 * m];
      const float keep = up ? v[c + 2 * m] : v[c];
      const float recv = __shfl_xor_sync(0xffffffffu, send, m);
      v[c] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return make_float2(v[0], v[1]);
}

// One persistent CTA per SM; warp 0 issues TMA loads, warp 1 the MMAs, warps
// 2-5 run the softmax.
//   S^T[t, h] = C[t, :] . q[h, :]      M = 64 rows, N = 64 heads, K = 576
//   O^T[d, h] += C[:, d]^T . P^T[:, h]  M = 128 latent dims (4 blocks), N = 64, K = 64
// Shared memory holds the resident q (72 KB) and two buffers of one 64 x 576
// tile each, as nine 8 KB boxes: the next tile streams into one buffer while
// the products and the softmax work on the other. A tile's boxes stay from
// its scores to its latent product; P^T is written into its rope box once
// the scores have read it.
// The tensor core takes about as long for an M = 64 as for an M = 128
// product and has a floor per instruction, so the issue order matters: the
// MMA warp issues the scores of tile j + 1 (into the second S^T buffer) as
// soon as that tile has landed, ahead of the latent product of tile j, which
// waits for the softmax; the tensor core then works through the softmax.
// The M = 64 score accumulator keeps row 16 q + i (i < 16) in TMEM lane
// 32 q + i: the softmax warp of lane quarter q reads its 16 rows with the
// two-halves load, a thread taking 32 of the 64 heads of one row. The
// softmax keeps a per-head reference max that it raises only when a score
// exceeds it by more than 8 (2^8 bounds P), so the common path needs one
// CTA-wide vote per tile and no column reduction.
__global__ void __launch_bounds__(kDecThreads, 1)
decode_attn_kernel(const __grid_constant__ CUtensorMap map_cache, const __grid_constant__ CUtensorMap map_q,
                   DecParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ DecBarriers bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();         // the schedule and the absorbed queries come from the previous kernel
  pdl_allow_next();
  const int c = blockIdx.x;
  const int64_t per = p.meta[0], total = p.meta[1];
  const int64_t r_lo = (int64_t)c * per;
  const int64_t r_hi = min(total, r_lo + per);
  if (r_lo >= r_hi) return;   // uniform over the CTA
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sBuf = smem + kDecQBytes;   // buffer b: box a at b * kDecBufBytes + a * kDecBoxBytes
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int b = 0; b < kDecBufs; ++b) { mbar_init(&bars.full[b], 1); mbar_init(&bars.empty[b], 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.s_full[b], 1);
      mbar_init(&bars.s_free[b], 128);
      mbar_init(&bars.p_full[b], 128);
    }
    mbar_init(&bars.pv_done[0], 1);
    mbar_init(&bars.pv_done[1], 1);
    mbar_init(&bars.o_free, 128);
    mbar_init(&bars.mma_done, 1);
    mbar_init(&bars.sm_sync, 128);
    bars.abort_flag = 0;
    mbar_fence_init();
  }
  if (threadIdx.x < kDecHeads) bars.m_ref[threadIdx.x] = -INFINITY;
  if (warp == 1) tmem_alloc(&bars.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    // tile j goes to buffer j & 1 once the latent product of tile j - 2 is done
    if (lane == 0) {
      tma_prefetch_desc(&map_cache);
      tma_prefetch_desc(&map_q);
      bool ok = true;
      int j = 0, nq = 0;   // tiles issued, q loads issued
      DecTileIter tiles, ahead;
      tiles.init(p, r_lo, r_hi);
      ahead.init(p, r_lo, r_hi);
      DecTile t, ta;
      // Tile j + 1 is prefetched into L2 when the copy of tile j is issued,
      // before its own buffer frees up: its copy into shared memory then
      // reads L2 instead of waiting on DRAM (a third tile in flight without
      // shared memory; prefetching further ahead measured slower).
      ahead.next(ta);
      while (ok && tiles.next(t)) {
        if (ahead.next(ta)) tma_prefetch_l2_3d(&map_cache, 0, (int)ta.row0, 0);
        if (t.first) {
          if (!mbar_wait(&bars.q_empty, ((uint32_t)t.seg & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.q_full, kDecQBytes);
          tma_load_3d(sQ, &map_q, &bars.q_full, 0, t.b * kDecHeads, 0);   // nine [64 heads x 64] blocks
          ++nq;
        }
        const int bj = j & 1;
        if (!mbar_wait(&bars.empty[bj], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t* buf = sBuf + bj * kDecBufBytes;
        mbar_arrive_expect_tx(&bars.full[bj], kDecBufBytes);
        tma_load_3d(buf, &map_cache, &bars.full[bj], 0, (int)t.row0, 0);   // nine [64 rows x 64] boxes
        ++j;
      }
      if (!ok) {   // let the copies in flight land before the CTA exits
        if (nq > 0) mbar_wait_drain(&bars.q_full, (uint32_t)(nq - 1) & 1u);
        for (int b = 0; b < kDecBufs; ++b) {
          const int n = (j + 1 - b) / 2;   // tiles j' < j with j' & 1 == b
          if (n > 0) mbar_wait_drain(&bars.full[b], (uint32_t)(n - 1) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    // Polls, in this order: the latent product of tile jo (its P^T written),
    // then the scores of tile js (its buffer landed, its S^T buffer read),
    // with js at most one tile ahead of jo. Decisions are warp-uniform.
    const uint32_t idesc_s = idesc_bf16_f32(kDecRows, kDecHeads);
    const uint32_t idesc_o = idesc_bf16_f32(128, kDecHeads) | kIdescAMajorMN | kIdescBMajorMN;
    DecTileIter its, ito;
    its.init(p, r_lo, r_hi);
    ito.init(p, r_lo, r_hi);
    DecTile ts, to;
    bool have_s = its.next(ts), have_o = ito.next(to);
    int js = 0, jo = 0;
    uint64_t t_idle = global_timer_ns();
    uint32_t spins = 0;
    while (have_o) {
      if (js > jo) {   // ---- O^T(jo) += C^T P^T ----
        bool ready = mbar_test(&bars.p_full[jo & 1], (uint32_t)(jo >> 1) & 1u);
        if (to.first && to.seg > 0) ready = ready && mbar_test(&bars.o_free, (uint32_t)(to.seg - 1) & 1u);
        if (__all_sync(0xffffffffu, ready)) {
          tc_fence_after();
          uint8_t* buf = sBuf + (jo & 1) * kDecBufBytes;
          const uint64_t pd = desc_mnmajor_sw128(smem_u32(buf + kDecLatBoxes * kDecBoxBytes), kDecBoxBytes, 1024);
          for (int blk = 0; blk < 4; ++blk) {
            // latent columns [128 blk, 128 blk + 128): boxes 2 blk, 2 blk + 1, read MN-major
            const uint64_t ad = desc_mnmajor_sw128(smem_u32(buf + 2 * blk * kDecBoxBytes), kDecBoxBytes, 1024);
#pragma unroll
            for (int k = 0; k < kDecRows / 16; ++k)
              mma_ss_elect(tmem + kDecOCol + blk * kDecHeads, desc_advance(ad, k * 2048),
                           desc_advance(pd, k * 2048), idesc_o, (to.first && k == 0) ? 0u : 1u);
          }
          mma_commit_elect(&bars.empty[jo & 1]);   // the buffer (and the P^T in it) is free
          mma_commit_elect(&bars.pv_done[jo & 1]);
          ++jo;
          have_o = ito.next(to);
          t_idle = global_timer_ns();
          continue;
        }
      }
      if (have_s && js <= jo + 1) {   // ---- S^T(js) ----
        const uint32_t u = (uint32_t)(js >> 1) & 1u;
        bool ready = mbar_test(&bars.full[js & 1], u) && mbar_test(&bars.s_free[js & 1], u ^ 1u);
        if (ts.first) ready = ready && mbar_test(&bars.q_full, (uint32_t)ts.seg & 1u);
        if (__all_sync(0xffffffffu, ready)) {
          tc_fence_after();
          uint8_t* buf = sBuf + (js & 1) * kDecBufBytes;
          const uint32_t sd = tmem + kDecSCol + (uint32_t)(js & 1) * kDecHeads;
          for (int a = 0; a < kDecBoxes; ++a) {
            const uint64_t cd = desc_kmajor_sw128(smem_u32(buf + a * kDecBoxBytes));
            const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + a * kDecHeads * 128));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_ss_elect(sd, desc_advance(cd, k * 32), desc_advance(qd, k * 32), idesc_s, (a | k) != 0);
          }
          mma_commit_elect(&bars.s_full[js & 1]);
          if (ts.last) mma_commit_elect(&bars.q_empty);   // q may be replaced once these are done
          ++js;
          have_s = its.next(ts);
          t_idle = global_timer_ns();
          continue;
        }
      }
      if ((++spins & 255u) == 0) {   // bounded: give up after kWaitLimitNs without progress
        bool stop = *abort_flag != 0;
        if (!stop && global_timer_ns() - t_idle > kWaitLimitNs) {
          if (lane == 0) { *abort_flag = 1; raise_device_error(kDevErrTimeout); }
          stop = true;
        }
        if (__any_sync(0xffffffffu, stop)) break;
      }
    }
    mma_commit_elect(&bars.mma_done);          // every MMA done before TMEM is freed
    if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
    __syncwarp();
  } else {
    // ---------------- softmax / correction / partial epilogue (warps 2-5) ----------------
    const int grp = warp & 3;                       // TMEM lane quarter
    const int tix = grp * 32 + lane;                // O^T latent row of this thread
    const int hh = lane >> 4;                       // scores of heads [32 hh, 32 hh + 32) ...
    const int row = grp * 16 + (lane & 15);         // ... of this tile row
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    int sync_ph = 0;
    auto cta_sync = [&]() -> bool {                 // bounded barrier of the 128 softmax threads
      mbar_arrive(&bars.sm_sync);
      const bool r = mbar_wait_warp(&bars.sm_sync, (uint32_t)sync_ph & 1u, abort_flag);
      ++sync_ph;
      return r;
    };
    float lpart[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) lpart[i] = 0.f;
    DecTileIter tiles;
    tiles.init(p, r_lo, r_hi);
    DecTile t;
    int j = 0;
    bool ok = true;
    while (ok && tiles.next(t)) {
      const int b2 = j & 1;
      uint8_t* sP = sBuf + (j & 1) * kDecBufBytes + kDecLatBoxes * kDecBoxBytes;   // P^T [64 rows x 64 heads]
      const uint32_t u = (uint32_t)(j >> 1) & 1u;
      if (!mbar_wait_warp(&bars.s_full[j & 1], u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float x[32];
      {
        uint32_t v[32];
        tmem_ld_halves32(tmem + lane_base + (uint32_t)(kDecSCol + (j & 1) * kDecHeads), v);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(v[i]);
      }
      tc_fence_before();
      mbar_arrive(&bars.s_free[j & 1]);
      const bool valid = row < t.nvalid;
      bool exceed = false;
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 mr = *reinterpret_cast<const float4*>(&bars.m_ref[32 * hh + q4 * 4]);
        const float mrv[4] = {mr.x, mr.y, mr.z, mr.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = q4 * 4 + e;
          const float xv = valid ? x[i] * p.scale_log2 : -INFINITY;
          x[i] = xv;
          exceed |= xv > mrv[e] + 8.f;
        }
      }
      const unsigned wv = __ballot_sync(0xffffffffu, exceed);
      if (lane == 0) bars.vote[b2][grp] = wv != 0u;
      if (!cta_sync()) { ok = false; break; }
      const bool any = (bars.vote[b2][0] | bars.vote[b2][1] | bars.vote[b2][2] | bars.vote[b2][3]) != 0;
      if (any) {
        // rare path: raise the reference max of heads whose scores outgrew it
        float tmp[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) tmp[i] = x[i];
        const float2 cm = half_column_reduce<true>(tmp, lane);
        bars.red[grp][32 * hh + 2 * (lane & 15)] = cm.x;
        bars.red[grp][32 * hh + 2 * (lane & 15) + 1] = cm.y;
        if (!cta_sync()) { ok = false; break; }
        if (tix < kDecHeads) {
          const float mo = bars.m_ref[tix];
          const float mt = fmaxf(fmaxf(bars.red[0][tix], bars.red[1][tix]), fmaxf(bars.red[2][tix], bars.red[3][tix]));
          float a = 1.f;
          if (mt > mo) {
            a = (mo == -INFINITY) ? 0.f : ex2_approx(mo - mt);
            bars.m_ref[tix] = mt;
          }
          bars.alpha[tix] = a;
        }
        if (!cta_sync()) { ok = false; break; }
#pragma unroll
        for (int i = 0; i < 32; ++i) lpart[i] *= bars.alpha[32 * hh + i];
        if (!t.first) {
          // O^T holds the segment's earlier tiles once the latent product of
          // tile j - 1 is done. Its barrier's previous phase (tile j - 3) is
          // complete, as is that of tile j - 2 (tile j's buffer was loaded
          // after it), and tile j + 1's is not issued: the parity is exact.
          if (!mbar_wait_warp(&bars.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int blk = 0; blk < 4; ++blk)
#pragma unroll 1
            for (int cc = 0; cc < kDecHeads / 16; ++cc) {
              uint32_t v[16];
              const uint32_t ta = tmem + lane_base + (uint32_t)(kDecOCol + blk * kDecHeads + cc * 16);
              tmem_ld16(ta, v);
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * bars.alpha[cc * 16 + e]);
              tmem_st16(ta, v);
            }
          tmem_st_wait();
        }
      }
      // this thread's half row of P^T (relative to the reference max), bf16, into the rope box
      uint32_t pk[16];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const float4 mr = *reinterpret_cast<const float4*>(&bars.m_ref[32 * hh + q4 * 4]);
        const uint32_t a0 = pack_bf16x2(ex2_approx(x[q4 * 4] - mr.x), ex2_approx(x[q4 * 4 + 1] - mr.y));
        const uint32_t a1 = pack_bf16x2(ex2_approx(x[q4 * 4 + 2] - mr.z), ex2_approx(x[q4 * 4 + 3] - mr.w));
        pk[q4 * 2] = a0;
        pk[q4 * 2 + 1] = a1;
        const float2 f0 = unpack_bf16x2(a0), f1 = unpack_bf16x2(a1);
        lpart[q4 * 4] += f0.x;
        lpart[q4 * 4 + 1] += f0.y;
        lpart[q4 * 4 + 2] += f1.x;
        lpart[q4 * 4 + 3] += f1.y;
      }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        *reinterpret_cast<uint4*>(sP + sw128_offset(row, 4 * hh + cc)) =
            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars.p_full[j & 1]);
      if (t.last) {
        // segment epilogue: unnormalized partial to slot (b + cta)
        const int slot = t.b + c;
        // the latent products of tiles j - 1 (which may still run: the
        // scores of tile j can be issued ahead of it) and j, each on the
        // barrier of its tile's parity. On either barrier the previous phase
        // (tile j - 3 or j - 2) is complete and the next (tile j + 1 or j + 2)
        // not issued, so each wait is at most one phase behind.
        if (j > 0 && !mbar_wait_warp(&bars.pv_done[(j - 1) & 1], (uint32_t)((j - 1) >> 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (!mbar_wait_warp(&bars.pv_done[j & 1], (uint32_t)(j >> 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk)
#pragma unroll 1
          for (int cc = 0; cc < kDecHeads / 16; ++cc) {
            uint32_t v[16];
            tmem_ld16(tmem + lane_base + (uint32_t)(kDecOCol + blk * kDecHeads + cc * 16), v);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              p.o_part[((int64_t)slot * p.H + cc * 16 + e) * p.R + blk * 128 + tix] = __uint_as_float(v[e]);
          }
        const float2 ls = half_column_reduce<false>(lpart, lane);
        bars.red[grp][32 * hh + 2 * (lane & 15)] = ls.x;
        bars.red[grp][32 * hh + 2 * (lane & 15) + 1] = ls.y;
        if (!cta_sync()) { ok = false; break; }
        if (tix < kDecHeads) {
          p.m_part[(int64_t)slot * p.H + tix] = bars.m_ref[tix];
          p.l_part[(int64_t)slot * p.H + tix] =
              bars.red[0][tix] + bars.red[1][tix] + bars.red[2][tix] + bars.red[3][tix];
          bars.m_ref[tix] = -INFINITY;   // the next segment starts afresh
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) lpart[i] = 0.f;
        if (!cta_sync()) { ok = false; break; }
        tc_fence_before();
        mbar_arrive(&bars.o_free);
      }
      ++j;
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
// b + c of the CTAs c whose ranges touch sequence b. One block per (b, 4
// heads), 8 latent values per thread; output bf16 (the MMA operand of the
// un-absorption).
__global__ void __launch_bounds__(256)
decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ m_part,
                      const float* __restrict__ l_part, const int64_t* __restrict__ prefix,
                      const int64_t* __restrict__ meta, int H, int R, __nv_bfloat16* __restrict__ o_lat) {
  pdl_wait();         // the partials come from the previous kernel
  pdl_allow_next();
  const int b = blockIdx.x;
  const int h = blockIdx.y * 4 + (threadIdx.x >> 6);
  const int d0 = (threadIdx.x & 63) * 8;
  if (h >= H || d0 >= R) return;
  const int64_t per = meta[0];
  const int64_t p0 = prefix[b], p1 = prefix[b + 1];
  uint4* dst = reinterpret_cast<uint4*>(o_lat + ((int64_t)b * H + h) * R + d0);
  if (p1 <= p0 || per <= 0) {   // a skipped sequence: no row to attend
    *dst = make_uint4(0, 0, 0, 0);
    return;
  }
  const int c0 = (int)(p0 / per), c1 = (int)((p1 - 1) / per);
  float M = -INFINITY;
  for (int cc = c0; cc <= c1; ++cc) M = fmaxf(M, m_part[(int64_t)(b + cc) * H + h]);
  float Lsum = 0.f, acc[8] = {};
  for (int cc = c0; cc <= c1; ++cc) {
    const int64_t slot = b + cc;
    const float ms = m_part[slot * H + h];
    if (ms == -INFINITY) continue;
    const float w = ex2_approx(ms - M);
    Lsum = fmaf(w, l_part[slot * H + h], Lsum);
    const float4* src = reinterpret_cast<const float4*>(o_part + (slot * H + h) * R + d0);
    const float4 a = src[0], bq = src[1];
    acc[0] = fmaf(w, a.x, acc[0]); acc[1] = fmaf(w, a.y, acc[1]);
    acc[2] = fmaf(w, a.z, acc[2]); acc[3] = fmaf(w, a.w, acc[3]);
    acc[4] = fmaf(w, bq.x, acc[4]); acc[5] = fmaf(w, bq.y, acc[5]);
    acc[6] = fmaf(w, bq.z, acc[6]); acc[7] = fmaf(w, bq.w, acc[7]);
  }
  const float inv = 1.f / Lsum;
  *dst = make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                    pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
}

// ---- per-head GEMM on tensor cores (q absorption, un-absorption) -----------------
// For head h (grid x), a block of 128 output features n (grid y) and a block of
// 64 batch rows b (grid z):   out[b, n] = sum_k A_h[n, k] Bm[b, k]
// A_h is a weight slice of kv_b_proj, Bm the per-head activations. On the
// tensor core it is D^T[n, b] = A[n, :] . Bm[b, :] with M = 128 (n), N = 64 (b):
//   kAMN = true : A is read MN-major (the weight stored [k][n]: W_UK_h), its
//                 TMA box [64 k x 64 n] twice per 64-wide K chunk;
//   kAMN = false: A is read K-major (the weight stored [n][k]: W_UV_h), its box
//                 [128 n x 64 k] per K chunk.
// Bm comes through a 3D map {K, H, B} as [64 b x 64 k] boxes. The output row
// of b is out[b * out_bs + h * out_hs + n]: bf16, or fp32 into out_f32 when
// that is set (the Linears whose result feeds an RMSNorm). kF16: both
// operands fp16 instead of bf16.
constexpr int kHgStages = 4;
constexpr int kHgABytes = 128 * 128;            // 128 n x 64 k bf16
constexpr int kHgBBytes = 64 * 128;             // 64 b x 64 k bf16
constexpr size_t kHgSmem = (size_t)kHgStages * (kHgABytes + kHgBBytes) + 1024;

struct HgParams {
  __nv_bfloat16* out;
  float* out_f32;        // when set: fp32 results here instead of `out`
  int64_t out_bs, out_hs;
  int B, Nout, K;
  int a_row0;            // first weight row of head h: a_row0 + h * a_hstride
  int a_hstride;
  // q absorption only: the CTAs of the first output block also rotate q_pe
  // into out[b, h, Nout:], and one extra CTA (x index H) builds the split
  // schedule of the attention
  const __nv_bfloat16* q;
  const int32_t* positions;
  const float* cos_t;
  const float* sin_t;
  int max_pos, N, interleaved;     // rotary width 64
  int qf_heads;                    // heads per sequence in the output rows (the padded count)
  const int32_t* lens;
  const int64_t* offsets;
  int max_len, G;
  int64_t cache_rows;
  int64_t* prefix;
  int64_t* meta;
};

template <bool kAMN, bool kF16 = false>
__global__ void __launch_bounds__(192, 1)
head_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b, HgParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ uint64_t full[kHgStages], empty[kHgStages], done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_allow_next();
  const int h = blockIdx.x, n0 = blockIdx.y * 128, b0 = blockIdx.z * 64;
  if (kAMN && h == (int)gridDim.x - 1) {   // the extra CTA column (uniform over the CTA)
    if (blockIdx.y == 0 && blockIdx.z == 0)
      decode_schedule_block(p.lens, p.offsets, p.B, p.max_len, p.cache_rows, p.G, p.prefix, p.meta);
    return;
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kHgStages * kHgABytes;
  const int nk = p.K / 64;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kHgStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(&done, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, 64);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int arow = p.a_row0 + h * p.a_hstride;
  if (warp == 0) {
    if (lane == 0) {
      int kc = 0;
      bool ok = true;
      auto load_a = [&](int k, int s) {
        uint8_t* a = sA + s * kHgABytes;
        if (kAMN) {   // rows k, columns n: two [64 k x 64 n] boxes
          tma_load_2d(a, &map_a, &full[s], n0, arow + k * 64);
          tma_load_2d(a + kHgABytes / 2, &map_a, &full[s], n0 + 64, arow + k * 64);
        } else {      // rows n, columns k: one [128 n x 64 k] box
          tma_load_2d(a, &map_a, &full[s], k * 64, arow + n0);
        }
      };
      // un-absorption: the weight halves of the first stages do not depend on
      // the previous kernel (o_lat does), so they load before the wait. (A
      // launch with programmatic serialization must therefore never follow
      // a kernel that writes the weight; the Linears launch the plain way.)
      const int npre = kAMN ? 0 : min(nk, kHgStages);
      for (int k = 0; k < npre; ++k) {
        mbar_arrive_expect_tx(&full[k], kHgABytes + kHgBBytes);
        load_a(k, k);
      }
      if (!kAMN) pdl_wait();
      for (; kc < nk; ++kc) {
        const int s = kc % kHgStages;
        if (kc >= npre) {
          if (!mbar_wait(&empty[s], ((uint32_t)(kc / kHgStages) & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], kHgABytes + kHgBBytes);
          load_a(kc, s);
        }
        tma_load_3d(sB + s * kHgBBytes, &map_b, &full[s], kc * 64, h, b0);
      }
      if (!ok)
        for (int i = (kc > kHgStages ? kc - kHgStages : 0); i < kc; ++i)
          mbar_wait_drain(&full[i % kHgStages], (uint32_t)(i / kHgStages) & 1u);
    }
  } else if (warp == 1) {
    // MMA issuer: whole warp, one elected lane issues
    const uint32_t idesc = (kF16 ? idesc_f16_f32(128, 64) : idesc_bf16_f32(128, 64)) | (kAMN ? kIdescAMajorMN : 0u);
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % kHgStages;
      if (!mbar_wait_warp(&full[s], (uint32_t)(kc / kHgStages) & 1u, &abort_flag)) break;
      tc_fence_after();
      const uint32_t aaddr = smem_u32(sA + s * kHgABytes);
      const uint64_t ad = kAMN ? desc_mnmajor_sw128(aaddr, kHgABytes / 2, 1024) : desc_kmajor_sw128(aaddr);
      const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + s * kHgBBytes));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_ss_elect(tmem, desc_advance(ad, kAMN ? k * 2048 : k * 32), desc_advance(bd, k * 32), idesc, (kc | k) != 0);
      mma_commit_elect(&empty[s]);
    }
    mma_commit_elect(&done);
    if (lane == 0) mbar_wait_drain(&done, 0);
    __syncwarp();
  } else {
    const int grp = warp & 3;
    const int n = n0 + grp * 32 + lane;
    if (mbar_wait_warp(&done, 0, &abort_flag)) {
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(grp * 32) << 16) + (uint32_t)(cc * 16), v);
        if (n < p.Nout) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int b = b0 + cc * 16 + e;
            const int64_t o = (int64_t)b * p.out_bs + (int64_t)h * p.out_hs + n;
            if (b < p.B) {
              if (p.out_f32) p.out_f32[o] = __uint_as_float(v[e]);
              else p.out[o] = __float2bfloat16_rn(__uint_as_float(v[e]));
            }
          }
        }
      }
    }
    if (kAMN && blockIdx.y == 0)
      decode_qrope_rows(p.q, p.positions, p.cos_t, p.sin_t, p.max_pos, h, b0, min(64, p.B - b0), gridDim.x - 1,
                        p.qf_heads, p.Nout, p.N, p.interleaved, p.out, threadIdx.x - 64);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

}  // namespace tc
}  // namespace mla
