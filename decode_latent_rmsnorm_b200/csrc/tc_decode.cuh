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
// Tensor-core mapping (M = 128 for both products, the shape tcgen05 runs at
// full rate; see decode_attn_kernel for the data flow):
//   S^T[t, h] : M = 128 cache rows, N = 64 heads, K = 576.
//   O^T[d, h] : M = 128 latent dims (4 blocks), N = 64 heads, K = 128 rows.
#pragma once
#include "tc_gemm.cuh"

namespace mla {
namespace tc {

constexpr int kDecRows = 128;                   // cache rows per tile (M of the score MMAs)
constexpr int kDecHeads = 64;                   // heads per CTA (N of both MMAs)
constexpr int kDecBoxes = 9;                    // 576 columns = 9 x 64
constexpr int kDecLatBoxes = 8;                 // the 512 latent columns
constexpr int kDecBoxBytes = kDecRows * 128;    // [128 rows x 64 cols] bf16 = 16 KB
constexpr int kDecSlots = kDecBoxes;            // one smem slot per box of a tile
constexpr int kDecQBytes = kDecBoxes * kDecHeads * 128;
constexpr int kDecPBytes = kDecRows * 128;      // P^T [128 rows x 64 heads] bf16
constexpr int kDecThreads = 192;
constexpr size_t kDecSmem = (size_t)kDecQBytes + kDecSlots * (size_t)kDecBoxBytes + 1024;   // P^T reuses the rope slot
constexpr int kDecOCol = 0;                     // O^T: 4 blocks x 64 columns
constexpr int kDecSCol = 256;                   // S^T: 64 columns

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
  uint64_t full[kDecSlots], empty[kDecSlots];
  uint64_t s_full, s_free;           // S^T (TMEM)
  uint64_t p_full, pv_done;          // P^T (smem, in the rope slot)
  uint64_t o_free, mma_done;
  uint64_t sm_sync;                  // bounded barrier of the 128 softmax threads
  uint32_t tmem_base;
  int abort_flag;
  int vote[2][4];                    // per tile parity: a vote is read after one sync, rewritten after two
  float m_ref[kDecHeads];            // per-head reference max (log2 units)
  float alpha[kDecHeads];
  float red[4][kDecHeads];           // per-warp column maxima / sums
};

// Column reduction of a warp: lane l holds v[0..63] (one value per head) and
// ends with the reduction over the warp's 32 lanes of heads 2l and 2l + 1
// (a halving exchange: 32 + 16 + 8 + 4 + 2 shuffles).
template <bool kMax>
__device__ __forceinline__ float2 warp_column_reduce(float (&v)[kDecHeads], int lane) {
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const bool up = lane & 16;
    const float send = up ? v[c] : v[c + 32];
    const float keep = up ? v[c + 32] : v[c];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 16);
    v[c] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const bool up = lane & 8;
    const float send = up ? v[c] : v[c + 16];
    const float keep = up ? v[c + 16] : v[c];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
    v[c] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const bool up = lane & 4;
    const float send = up ? v[c] : v[c + 8];
    const float keep = up ? v[c + 8] : v[c];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 4);
    v[c] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const bool up = lane & 2;
    const float send = up ? v[c] : v[c + 4];
    const float keep = up ? v[c + 4] : v[c];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
    v[c] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const bool up = lane & 1;
    const float send = up ? v[c] : v[c + 2];
    const float keep = up ? v[c + 2] : v[c];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    v[c] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
  return make_float2(v[0], v[1]);
}

// One persistent CTA per SM; warp 0 issues TMA loads, warp 1 the MMAs, warps
// 2-5 run the softmax (one cache row per thread: S^T lane = row).
//   S^T[t, h] = C[t, :] . q[h, :]      M = 128 rows, N = 64 heads, K = 576
//   O^T[d, h] += C[:, d]^T . P^T[:, h]  M = 128 latent dims (4 blocks), N = 64, K = 128
// Shared memory holds the resident q (72 KB) and one 128 x 576 tile as nine
// 16 KB boxes, one slot per box. The 8 latent boxes stay from the scores to
// the latent product; P^T is written into the rope box's slot once the
// scores have read it. Slots free up block by block as the latent product
// retires, and the next tile's boxes stream into them right away. The
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
  uint8_t* sSlot = smem + kDecQBytes;                       // slot a holds box a of the current tile
  uint8_t* sP = sSlot + (kDecSlots - 1) * kDecBoxBytes;     // P^T [128 rows x 64 heads] in the rope slot
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int a = 0; a < kDecSlots; ++a) { mbar_init(&bars.full[a], 1); mbar_init(&bars.empty[a], 1); }
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.s_free, 128);
    mbar_init(&bars.p_full, 128);
    mbar_init(&bars.pv_done, 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&map_cache);
      tma_prefetch_desc(&map_q);
      bool ok = true;
      int j = 0;
      DecTileIter tiles;
      tiles.init(p, r_lo, r_hi);
      DecTile t;
      while (ok && tiles.next(t)) {
        if (t.first) {
          if (!mbar_wait(&bars.q_empty, ((uint32_t)t.seg & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.q_full, kDecQBytes);
          for (int a = 0; a < kDecBoxes; ++a)
            tma_load_2d(sQ + a * kDecHeads * 128, &map_q, &bars.q_full, a * 64, t.b * kDecHeads);
        }
        for (int a = 0; a < kDecBoxes; ++a) {   // latent boxes first: they free up first
          if (!mbar_wait(&bars.empty[a], ((uint32_t)j & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.full[a], kDecBoxBytes);
          tma_load_2d(sSlot + a * kDecBoxBytes, &map_cache, &bars.full[a], a * 64, (int)t.row0);
        }
        ++j;
      }
      if (!ok) {   // let the copies in flight land before the CTA exits
        mbar_wait_drain(&bars.q_full, 0);
        for (int a = 0; a < kDecSlots; ++a) mbar_wait_drain(&bars.full[a], (uint32_t)(j > 0 ? j - 1 : 0) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    const uint32_t idesc_s = idesc_bf16_f32(kDecRows, kDecHeads);
    const uint32_t idesc_o = idesc_bf16_f32(128, kDecHeads) | kIdescAMajorMN | kIdescBMajorMN;
    bool ok = true;
    int j = 0;
    DecTileIter tiles;
    tiles.init(p, r_lo, r_hi);
    DecTile t;
    while (ok && tiles.next(t)) {
      const uint32_t ph = (uint32_t)j & 1u;
      // ---- S^T(j) ----
      if (t.first && !(ok = mbar_wait_warp(&bars.q_full, (uint32_t)t.seg & 1u, abort_flag))) break;
      if (!(ok = mbar_wait_warp(&bars.s_free, ph ^ 1u, abort_flag))) break;
      tc_fence_after();
      for (int a = 0; a < kDecBoxes && ok; ++a) {
        if (!(ok = mbar_wait_warp(&bars.full[a], ph, abort_flag))) break;
        tc_fence_after();
        const uint64_t cd = desc_kmajor_sw128(smem_u32(sSlot + a * kDecBoxBytes));
        const uint64_t qd = desc_kmajor_sw128(smem_u32(sQ + a * kDecHeads * 128));
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ss_elect(tmem + kDecSCol, desc_advance(cd, k * 32), desc_advance(qd, k * 32), idesc_s, (a | k) != 0);
      }
      if (!ok) break;
      mma_commit_elect(&bars.s_full);
      if (t.last) mma_commit_elect(&bars.q_empty);     // q may be replaced once these are done
      // ---- O^T(j) += C^T P^T ----
      if (t.first && t.seg > 0 && !(ok = mbar_wait_warp(&bars.o_free, (uint32_t)(t.seg - 1) & 1u, abort_flag))) break;
      if (!(ok = mbar_wait_warp(&bars.p_full, ph, abort_flag))) break;
      tc_fence_after();
      const uint64_t pd = desc_mnmajor_sw128(smem_u32(sP), kDecBoxBytes, 1024);
      for (int blk = 0; blk < 4; ++blk) {
        // latent columns [128 blk, 128 blk + 128): slots 2 blk, 2 blk + 1, read MN-major
        const uint64_t ad = desc_mnmajor_sw128(smem_u32(sSlot + 2 * blk * kDecBoxBytes), kDecBoxBytes, 1024);
#pragma unroll
        for (int k = 0; k < kDecRows / 16; ++k)
          mma_ss_elect(tmem + kDecOCol + blk * kDecHeads, desc_advance(ad, k * 2048), desc_advance(pd, k * 2048),
                       idesc_o, (t.first && k == 0) ? 0u : 1u);
        mma_commit_elect(&bars.empty[2 * blk]);
        mma_commit_elect(&bars.empty[2 * blk + 1]);
      }
      mma_commit_elect(&bars.empty[kDecSlots - 1]);    // P^T read: the rope slot is free
      mma_commit_elect(&bars.pv_done);
      ++j;
    }
    mma_commit_elect(&bars.mma_done);          // every MMA done before TMEM is freed
    if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
    __syncwarp();
  } else {
    // ---------------- softmax / correction / partial epilogue (warps 2-5) ----------------
    const int grp = warp & 3;                       // TMEM quadrant
    const int tix = grp * 32 + lane;                // cache row of the tile == O^T latent row
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    int sync_ph = 0;
    auto cta_sync = [&]() -> bool {                 // bounded barrier of the 128 softmax threads
      mbar_arrive(&bars.sm_sync);
      const bool r = mbar_wait_warp(&bars.sm_sync, (uint32_t)sync_ph & 1u, abort_flag);
      ++sync_ph;
      return r;
    };
    float lpart[kDecHeads];
#pragma unroll
    for (int h = 0; h < kDecHeads; ++h) lpart[h] = 0.f;
    DecTileIter tiles;
    tiles.init(p, r_lo, r_hi);
    DecTile t;
    int j = 0;
    bool ok = true;
    while (ok && tiles.next(t)) {
      const int b2 = j & 1;
      if (!mbar_wait_warp(&bars.s_full, (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float x[kDecHeads];
      {   // the row's 64 scores: two loads in flight, one wait
        uint32_t v[kDecHeads];
#pragma unroll
        for (int cc = 0; cc < kDecHeads / 32; ++cc)
          tmem_ld32_nowait(tmem + lane_base + (uint32_t)(kDecSCol + cc * 32), v + cc * 32);
        tmem_wait_ld64(v);
#pragma unroll
        for (int h = 0; h < kDecHeads; ++h) x[h] = __uint_as_float(v[h]);
      }
      tc_fence_before();
      mbar_arrive(&bars.s_free);
      const bool valid = tix < t.nvalid;
      bool exceed = false;
#pragma unroll
      for (int q4 = 0; q4 < kDecHeads / 4; ++q4) {
        const float4 mr = *reinterpret_cast<const float4*>(&bars.m_ref[q4 * 4]);
        const float mrv[4] = {mr.x, mr.y, mr.z, mr.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = q4 * 4 + e;
          const float xv = valid ? x[h] * p.scale_log2 : -INFINITY;
          x[h] = xv;
          exceed |= xv > mrv[e] + 8.f;
        }
      }
      const unsigned wv = __ballot_sync(0xffffffffu, exceed);
      if (lane == 0) bars.vote[b2][grp] = wv != 0u;
      if (!cta_sync()) { ok = false; break; }
      const bool any = (bars.vote[b2][0] | bars.vote[b2][1] | bars.vote[b2][2] | bars.vote[b2][3]) != 0;
      if (any) {
        // rare path: raise the reference max of heads whose scores outgrew it
        float tmp[kDecHeads];
#pragma unroll
        for (int h = 0; h < kDecHeads; ++h) tmp[h] = x[h];
        const float2 cm = warp_column_reduce<true>(tmp, lane);
        bars.red[grp][2 * lane] = cm.x;
        bars.red[grp][2 * lane + 1] = cm.y;
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
        for (int h = 0; h < kDecHeads; ++h) lpart[h] *= bars.alpha[h];
        if (!t.first) {
          // O^T holds the segment's earlier tiles (their P V finished before S^T(j) began)
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
      // P^T row of this thread (relative to the reference max), bf16, into the rope slot
      uint32_t pk[kDecHeads / 2];
#pragma unroll
      for (int q4 = 0; q4 < kDecHeads / 4; ++q4) {
        const float4 mr = *reinterpret_cast<const float4*>(&bars.m_ref[q4 * 4]);
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
      for (int cc = 0; cc < 8; ++cc)
        *reinterpret_cast<uint4*>(sP + sw128_offset(tix, cc)) =
            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars.p_full);
      if (t.last) {
        // segment epilogue: unnormalized partial to slot (b + cta)
        const int slot = t.b + c;
        if (!mbar_wait_warp(&bars.pv_done, (uint32_t)j & 1u, abort_flag)) { ok = false; break; }
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
        const float2 ls = warp_column_reduce<false>(lpart, lane);
        bars.red[grp][2 * lane] = ls.x;
        bars.red[grp][2 * lane + 1] = ls.y;
        if (!cta_sync()) { ok = false; break; }
        if (tix < kDecHeads) {
          p.m_part[(int64_t)slot * p.H + tix] = bars.m_ref[tix];
          p.l_part[(int64_t)slot * p.H + tix] =
              bars.red[0][tix] + bars.red[1][tix] + bars.red[2][tix] + bars.red[3][tix];
          bars.m_ref[tix] = -INFINITY;   // the next segment starts afresh
        }
#pragma unroll
        for (int h = 0; h < kDecHeads; ++h) lpart[h] = 0.f;
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
