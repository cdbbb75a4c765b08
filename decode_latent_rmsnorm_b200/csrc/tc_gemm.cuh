// Tensor-core (tcgen05) prefill front half: tile schedule of the packed
// sequences, and the fused latent RMSNorm + kv_b_proj up-projection.
//
// Sources: "Eager latent expansion" equation page (normalize the compressed
// latent, apply the learned up-projection, reshape into heads, split into
// non-rotary key and value); Kimi-K2 "RoPE coefficients" page, "Key heads"
// (mla-kv: split the joint latent into the 512-wide latent and k_pe, view
// k_pe as one head shared by all heads).
//
// Precision: the normalized latent c_hat = w * x / rms(x) is formed in fp32
// and handed to the tensor cores in fp16 (11 significant bits), against an
// fp16 copy of the weight (exact for weights in fp16's normal range), with
// fp32 accumulation; the values are stored in fp16 and k_nope in bf16 (the
// attention's non-rotary score atoms take q as given, in bf16). A value
// beyond the fp16 range sets the device error word.
//
// Workspace layout ("padded token space"): every sequence starts on a
// 128-row boundary, so a 128-token tile never straddles two sequences and
// every TMA coordinate along tokens is a multiple of 64 elements. Rows past a
// sequence's end are written as zeros.
//   k_nope [H, Tpad, N]  bf16   (row tp, N contiguous)
//   vt     [H, V, Tpad]  fp16   (values transposed: tokens contiguous)
//   k_rot  [Tpad, P]     fp16   (the shared rotary key, rotated)
#pragma once
#include "tc_ptx.cuh"

namespace mla {
namespace tc {

constexpr int kTile = 128;            // token rows per tile (M of the MMAs)

// ---- tile schedule --------------------------------------------------------
// tile_seq[i] / tile_q0[i]: sequence and first in-sequence row of tile i in
// natural order (padded rows tp = 128 i ...); order[j]: tiles sorted by
// decreasing causal work (largest q0 first), for the attention grid.
// pair_order[j]: the first tile of each 256-row block (tiles 2k and 2k + 1 of
// one sequence; the second may not exist), blocks sorted by decreasing k.
// Entries past the real tile / block count are -1. Bad cu_seqlens set the
// device error word and leave every entry at -1. item_counter (the two-tile
// attention's work counter) is reset to 0.
// Inclusive prefix sum over the 1024 threads of a block (thread order):
// a shuffle scan inside each warp, then one over the 32 warp totals.
// Every thread of the block must call it.
__device__ __forceinline__ int block_inclusive_scan_1024(int v, int* s_warp /* [32] */) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  __syncthreads();                       // s_warp free from any earlier use
  if (lane == 31) s_warp[wid] = v;
  __syncthreads();
  int w = s_warp[lane];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, w, o);
    if (lane >= o) w += y;
  }
  const int before = __shfl_sync(0xffffffffu, w, (wid + 31) & 31);   // total of the earlier warps
  return v + (wid > 0 ? before : 0);
}

// Largest sequence count whose bounds the schedule keeps in shared memory.
constexpr int kSchedSmemSeqs = 2048;

// Run by one block of 1024 threads.
__device__ __forceinline__ void schedule_block(const int32_t* __restrict__ cu, int nseq, int64_t Ttot,
                                               int max_seqlen, int cap, int32_t* __restrict__ seq_tile0,
                                               int32_t* __restrict__ tile_seq, int32_t* __restrict__ tile_q0,
                                               int32_t* __restrict__ order, int32_t* __restrict__ pair_order,
                                               int32_t* __restrict__ item_counter) {
  constexpr int kBuckets = 2048;   // = 2 * blockDim.x (launched with 1024 threads)
  __shared__ int s_bad;
  __shared__ int s_carry;
  __shared__ int s_scan[1024];
  __shared__ int s_cnt[kBuckets];
  __shared__ int s_off[kBuckets];
  const int tid = threadIdx.x;
  if (nseq <= kSchedSmemSeqs) {
    // fast path: cu_seqlens is read once into shared memory and every table
    // is derived there (each of the general path's dependent global round
    // trips costs a memory latency on the prefill's critical path)
    __shared__ int s_t0[kSchedSmemSeqs + 1];     // first tile of each sequence
    if (tid == 0) { s_bad = 0; s_carry = 0; *item_counter = 0; }
    for (int k = tid; k < kBuckets; k += blockDim.x) { s_cnt[k] = 0; s_off[k] = 0; }
    __syncthreads();
    // per-sequence tile counts (1024 sequences per pass) -> exclusive scan
    for (int base = 0; base < nseq; base += blockDim.x) {
      const int sq = base + tid;
      int n_here = 0;
      if (sq < nseq) {
        const int64_t a = cu[sq], b = cu[sq + 1];
        if (a < 0 || b < a || b > Ttot || b - a > max_seqlen) s_bad = 1;
        else n_here = (int)((b - a + kTile - 1) / kTile);
      }
      const int inc = block_inclusive_scan_1024(n_here, s_scan);
      if (sq < nseq) s_t0[sq] = s_carry + inc - n_here;
      __syncthreads();
      if (tid == (int)blockDim.x - 1) s_carry += inc;
      __syncthreads();
    }
    if (tid == 0) s_t0[nseq] = s_carry;
    __syncthreads();
    const int total = s_t0[nseq];
    if (s_bad || total > cap) {
      for (int i = tid; i < cap; i += blockDim.x) { tile_seq[i] = -1; tile_q0[i] = -1; order[i] = -1; pair_order[i] = -1; }
      if (tid == 0) raise_device_error(kDevErrBadInput);
      return;
    }
    for (int i = tid; i <= nseq; i += blockDim.x) seq_tile0[i] = s_t0[i];
    // tiles in natural order; bucket counts of causal work (tile index in
    // its sequence) for single tiles and for 256-row blocks. Every entry of
    // pair_order starts at -1 here: the blocks fill only its first entries
    // (one per two tiles), after the barriers below.
    for (int t = tid; t < cap; t += blockDim.x) {
      pair_order[t] = -1;
      if (t >= total) { tile_seq[t] = -1; tile_q0[t] = -1; order[t] = -1; continue; }
      int lo = 0, hi = nseq - 1;               // the sequence whose tiles hold t
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_t0[mid] <= t) lo = mid;
        else hi = mid - 1;
      }
      const int k = t - s_t0[lo];
      tile_seq[t] = lo;
      tile_q0[t] = k * kTile;
      atomicAdd(&s_cnt[min(k, kBuckets - 1)], 1);
    }
    __syncthreads();
    {
      const int k0 = kBuckets - 1 - 2 * tid, k1 = k0 - 1;
      const int c0 = s_cnt[k0], c1 = s_cnt[k1];
      const int before = block_inclusive_scan_1024(c0 + c1, s_scan) - (c0 + c1);
      s_off[k0] = before;
      s_off[k1] = before + c0;
    }
    __syncthreads();
    for (int t = tid; t < total; t += blockDim.x) {
      int lo = 0, hi = nseq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_t0[mid] <= t) lo = mid;
        else hi = mid - 1;
      }
      const int pos = atomicAdd(&s_off[min(t - s_t0[lo], kBuckets - 1)], 1);
      order[pos] = t;
    }
    __syncthreads();
    for (int k = tid; k < kBuckets; k += blockDim.x) s_cnt[k] = 0;
    __syncthreads();
    for (int t = tid; t < total; t += blockDim.x) {
      int lo = 0, hi = nseq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_t0[mid] <= t) lo = mid;
        else hi = mid - 1;
      }
      const int k = t - s_t0[lo];
      if ((k & 1) == 0) atomicAdd(&s_cnt[min(k / 2, kBuckets - 1)], 1);
    }
    __syncthreads();
    {
      const int k0 = kBuckets - 1 - 2 * tid, k1 = k0 - 1;
      const int c0 = s_cnt[k0], c1 = s_cnt[k1];
      const int before = block_inclusive_scan_1024(c0 + c1, s_scan) - (c0 + c1);
      s_off[k0] = before;
      s_off[k1] = before + c0;
    }
    __syncthreads();
    for (int t = tid; t < total; t += blockDim.x) {
      int lo = 0, hi = nseq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_t0[mid] <= t) lo = mid;
        else hi = mid - 1;
      }
      const int k = t - s_t0[lo];
      if ((k & 1) == 0) pair_order[atomicAdd(&s_off[min(k / 2, kBuckets - 1)], 1)] = t;
    }
    return;
  }
  if (tid == 0) { s_bad = 0; s_carry = 0; *item_counter = 0; }
  for (int i = tid; i < cap; i += blockDim.x) {
    tile_seq[i] = -1; tile_q0[i] = -1; order[i] = -1; pair_order[i] = -1;
  }
  for (int k = tid; k < kBuckets; k += blockDim.x) { s_cnt[k] = 0; s_off[k] = 0; }
  __syncthreads();
  // 1) per-sequence tile counts -> exclusive scan into seq_tile0
  for (int base = 0; base <= nseq; base += blockDim.x) {
    const int s = base + tid;
    int nt = 0;
    if (s < nseq) {
      const int64_t a = cu[s], b = cu[s + 1];
      if (a < 0 || b < a || b > Ttot || b - a > max_seqlen) s_bad = 1;
      else nt = (int)((b - a + kTile - 1) / kTile);
    }
    const int inc = block_inclusive_scan_1024(nt, s_scan);
    if (s <= nseq) seq_tile0[s] = s_carry + inc - nt;
    __syncthreads();
    if (tid == (int)blockDim.x - 1) s_carry += inc;
    __syncthreads();
  }
  if (s_bad) {
    if (tid == 0) raise_device_error(kDevErrBadInput);
    return;
  }
  if (s_carry > cap) {   // cannot happen for valid input; guards the arrays
    if (tid == 0) raise_device_error(kDevErrBadInput);
    return;
  }
  __syncthreads();
  // 2) tiles in natural order; 3) bucket counts of causal work (tile index)
  for (int s = tid; s < nseq; s += blockDim.x) {
    const int t0 = seq_tile0[s], nt = seq_tile0[s + 1] - t0;
    for (int k = 0; k < nt; ++k) {
      tile_seq[t0 + k] = s;
      tile_q0[t0 + k] = k * kTile;
      atomicAdd(&s_cnt[min(k, kBuckets - 1)], 1);
    }
  }
  __syncthreads();
  {
    // descending exclusive offsets: s_off[k] = sum of s_cnt[k'] for k' > k.
    // Thread i owns reversed buckets 2i and 2i + 1 (bucket kBuckets-1-2i, ...).
    const int k0 = kBuckets - 1 - 2 * tid, k1 = k0 - 1;
    const int c0 = s_cnt[k0], c1 = s_cnt[k1];
    const int before = block_inclusive_scan_1024(c0 + c1, s_scan) - (c0 + c1);
    s_off[k0] = before;
    s_off[k1] = before + c0;
  }
  __syncthreads();
  for (int s = tid; s < nseq; s += blockDim.x) {
    const int t0 = seq_tile0[s], nt = seq_tile0[s + 1] - t0;
    for (int k = 0; k < nt; ++k) {
      const int pos = atomicAdd(&s_off[min(k, kBuckets - 1)], 1);
      order[pos] = t0 + k;
    }
  }
  // 4) the same for 256-row blocks, bucketed by block index
  __syncthreads();
  for (int k = tid; k < kBuckets; k += blockDim.x) s_cnt[k] = 0;
  __syncthreads();
  for (int s = tid; s < nseq; s += blockDim.x) {
    const int nt = seq_tile0[s + 1] - seq_tile0[s];
    for (int k = 0; k < nt; k += 2) atomicAdd(&s_cnt[min(k / 2, kBuckets - 1)], 1);
  }
  __syncthreads();
  {
    const int k0 = kBuckets - 1 - 2 * tid, k1 = k0 - 1;
    const int c0 = s_cnt[k0], c1 = s_cnt[k1];
    const int before = block_inclusive_scan_1024(c0 + c1, s_scan) - (c0 + c1);
    s_off[k0] = before;
    s_off[k1] = before + c0;
  }
  __syncthreads();
  for (int s = tid; s < nseq; s += blockDim.x) {
    const int t0 = seq_tile0[s], nt = seq_tile0[s + 1] - t0;
    for (int k = 0; k < nt; k += 2) {
      const int pos = atomicAdd(&s_off[min(k / 2, kBuckets - 1)], 1);
      pair_order[pos] = t0 + k;
    }
  }
}

// ---- prefill preparation: tile schedule, fp16 weight, normalized latent ----
// Block 0 builds the schedule (schedule_block); blocks 1 .. w_blocks convert
// the weight, kPrepUnroll x 8 values per thread; the next norm_blocks (when
// launched) write the normalized latent in fp16 for the transposed-value
// GEMM, and the blocks after those the rotated query rows (q_rope_warp,
// four warps per token). A value beyond the fp16 range sets the device error
// word.
constexpr int kPrepThreads = 1024;
constexpr int kPrepUnroll = 8;

// The rotary part of every query head, turned at its token's position once
// for all key steps: qr [Ttot, H, 64] fp16 (the attention kernels' last
// score atom). Source: Kimi-K2 "RoPE coefficients" page, "Query heads": each
// head's rotary query part is rotated at the token's position like the key's.
struct QRopeParams {
  const __nv_bfloat16* q;       // [Ttot, H, D], the rotary part in columns N .. N + 63
  const int32_t* positions;     // [Ttot]
  const float* cos_t;           // [max_pos, 32]
  const float* sin_t;
  __half* qr;                   // [Ttot, H, 64]
  int64_t rows;                 // Ttot * H
  int H, D, N, max_pos, interleaved;
};

// The rotation runs one token per group of kQrWarpsPerToken warps: the
// token's position and its cosine / sine row are read once by each warp, and
// lane l of a warp turns the pairs 2 (l & 15) and 2 (l & 15) + 1 of the heads
// h = 8 k + 2 w + (l >> 4) (w the warp of the token, k = 0, 1, ...): pair i
// is (x_i, x_{i+32}) (half-split) or (x_{2i}, x_{2i+1}) (interleaved), turned
// by the angle of pair i at positions[t], each result rounded once to fp16.
// Four heads of a lane have their loads in flight together. A value beyond
// the fp16 range sets the device error word.
constexpr int kQrWarpsPerToken = 4;
__device__ __forceinline__ void q_rope_warp(const QRopeParams& p, int64_t w, int lane) {
  const int64_t T = p.rows / p.H;
  const int64_t t = w / kQrWarpsPerToken;
  if (t >= T) return;
  const int wq = (int)(w % kQrWarpsPerToken), hs = lane >> 4, l = lane & 15;
  const int64_t pos = checked_pos(p.positions[t], p.max_pos);
  const float2 cs = *reinterpret_cast<const float2*>(p.cos_t + pos * 32 + 2 * l);
  const float2 sn = *reinterpret_cast<const float2*>(p.sin_t + pos * 32 + 2 * l);
  const int nk = (p.H + 7) / 8;
  float mx = 0.f;
  for (int k0 = 0; k0 < nk; k0 += 4) {
    uint32_t ra[4], rb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = 8 * (k0 + u) + 2 * wq + hs;
      if (h < p.H) {
        const __nv_bfloat16* src = p.q + (t * p.H + h) * p.D + p.N;
        if (p.interleaved) {
          const uint2 v = *reinterpret_cast<const uint2*>(src + 4 * l);
          ra[u] = v.x;
          rb[u] = v.y;
        } else {
          ra[u] = *reinterpret_cast<const uint32_t*>(src + 2 * l);
          rb[u] = *reinterpret_cast<const uint32_t*>(src + 32 + 2 * l);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int h = 8 * (k0 + u) + 2 * wq + hs;
      if (h >= p.H) continue;
      const float2 a = unpack_bf16x2(ra[u]), b = unpack_bf16x2(rb[u]);
      __half* dst = p.qr + (t * p.H + h) * 64;
      float y0, y1, y2, y3;
      if (p.interleaved) {   // pairs (a.x, a.y) and (b.x, b.y)
        rope_turn(a.x, a.y, cs.x, sn.x, y0, y1);
        rope_turn(b.x, b.y, cs.y, sn.y, y2, y3);
        *reinterpret_cast<uint2*>(dst + 4 * l) = make_uint2(pack_f16x2(y0, y1), pack_f16x2(y2, y3));
      } else {               // pairs (a.x, b.x) and (a.y, b.y)
        rope_turn(a.x, b.x, cs.x, sn.x, y0, y2);
        rope_turn(a.y, b.y, cs.y, sn.y, y1, y3);
        *reinterpret_cast<uint32_t*>(dst + 2 * l) = pack_f16x2(y0, y1);
        *reinterpret_cast<uint32_t*>(dst + 32 + 2 * l) = pack_f16x2(y2, y3);
      }
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(y0), fabsf(y1)), fmaxf(fabsf(y2), fabsf(y3))));
    }
  }
  if (!(mx <= kF16Max)) raise_device_error(kDevErrRange);
}
// Blocks of the rotation for `rows` = tokens x heads.
__host__ __device__ constexpr int64_t q_rope_blocks(int64_t rows, int H, int threads) {
  return (rows / H * kQrWarpsPerToken * 32 + threads - 1) / threads;
}

// The rotated query rows on their own (chunks over a cached prefix, whose
// positions the previous kernel writes).
__global__ void __launch_bounds__(kPrepThreads)
q_rope_kernel(QRopeParams p) {
  pdl_wait();
  pdl_allow_next();
  q_rope_warp(p, ((int64_t)blockIdx.x * kPrepThreads + threadIdx.x) >> 5, (int)(threadIdx.x & 31));
}

// Block `blk` of the fp16 weight copy: kPrepUnroll x 8 values per thread
// (n8 groups of 8 values in all). A value beyond the fp16 range sets the
// device error word.
__device__ __forceinline__ void weight_f16_block(const __nv_bfloat16* __restrict__ w, __half* __restrict__ w16,
                                                 int64_t n8, int64_t blk) {
  const int64_t base = blk * kPrepThreads * kPrepUnroll + threadIdx.x;
  uint4 v[kPrepUnroll];
#pragma unroll
  for (int u = 0; u < kPrepUnroll; ++u) {
    const int64_t i = base + (int64_t)u * kPrepThreads;
    if (i < n8) v[u] = reinterpret_cast<const uint4*>(w)[i];
  }
  float mx = 0.f;
#pragma unroll
  for (int u = 0; u < kPrepUnroll; ++u) {
    const int64_t i = base + (int64_t)u * kPrepThreads;
    if (i >= n8) break;
    const uint32_t in[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(in[e]);
      mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      o[e] = pack_f16x2(f.x, f.y);
    }
    reinterpret_cast<uint4*>(w16)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (!(mx <= kF16Max)) raise_device_error(kDevErrRange);
}
__global__ void __launch_bounds__(kPrepThreads)
prefill_prep_kernel(const int32_t* __restrict__ cu, int nseq, int64_t Ttot, int max_seqlen, int cap,
                    int32_t* __restrict__ seq_tile0, int32_t* __restrict__ tile_seq,
                    int32_t* __restrict__ tile_q0, int32_t* __restrict__ order, int32_t* __restrict__ pair_order,
                    int32_t* __restrict__ item_counter,
                    const __nv_bfloat16* __restrict__ w, __half* __restrict__ w16, int64_t n8, int w_blocks,
                    const __nv_bfloat16* __restrict__ latent, const __nv_bfloat16* __restrict__ w_norm, int R,
                    float eps, __half* __restrict__ c16, int norm_blocks, QRopeParams qrp) {
  pdl_allow_next();
  if (blockIdx.x == 0) {
    schedule_block(cu, nseq, Ttot, max_seqlen, cap, seq_tile0, tile_seq, tile_q0, order, pair_order,
                   item_counter);
    return;
  }
  if ((int)blockIdx.x > w_blocks + norm_blocks) {
    q_rope_warp(qrp, ((int64_t)((int)blockIdx.x - 1 - w_blocks - norm_blocks) * kPrepThreads + threadIdx.x) >> 5,
                (int)(threadIdx.x & 31));
    return;
  }
  if ((int)blockIdx.x > w_blocks) {
    // normalized latent c_hat = w * x / sqrt(mean(x^2) + eps) in fp16
    // [Ttot, R]: one warp per token row; lane l holds the 8-value chunks l and
    // l + 32 of the row (R <= 512)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)((int)blockIdx.x - 1 - w_blocks) * (kPrepThreads / 32) + warp;
    if (t >= Ttot) return;
    const int nch = R / 8;
    const uint4* src = reinterpret_cast<const uint4*>(latent + t * (R + 64));
    const uint4* wn = reinterpret_cast<const uint4*>(w_norm);
    uint4 xv[2], gv[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int c = lane + 32 * k;
      xv[k] = c < nch ? src[c] : make_uint4(0u, 0u, 0u, 0u);
      gv[k] = c < nch ? wn[c] : make_uint4(0u, 0u, 0u, 0u);
    }
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w4[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 v = unpack_bf16x2(w4[e]);
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, ss));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss / (float)R + eps);
    float mx = 0.f;
    uint4* dst = reinterpret_cast<uint4*>(c16 + t * R);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int c = lane + 32 * k;
      if (c >= nch) break;
      const uint32_t w4[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
      const uint32_t g4[4] = {gv[k].x, gv[k].y, gv[k].z, gv[k].w};
      uint32_t o4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 v = unpack_bf16x2(w4[e]);
        const float2 g = unpack_bf16x2(g4[e]);
        const float a = g.x * (v.x * r), b = g.y * (v.y * r);
        mx = fmaxf(mx, fmaxf(fabsf(a), fabsf(b)));
        o4[e] = pack_f16x2(a, b);
      }
      dst[c] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
    if (!(mx <= kF16Max)) raise_device_error(kDevErrRange);
    return;
  }
  weight_f16_block(w, w16, n8, (int64_t)(blockIdx.x - 1));
}

// The fp16 copy of kv_b_proj on its own (mla_prepare_kv_b_proj), one block
// per kPrepThreads x kPrepUnroll groups of 8 values.
__global__ void __launch_bounds__(kPrepThreads)
weight_f16_kernel(const __nv_bfloat16* __restrict__ w, __half* __restrict__ w16, int64_t n8) {
  weight_f16_block(w, w16, n8, (int64_t)blockIdx.x);
}

// ---- fused RMSNorm + kv_b_proj GEMM ------------------------------------------
constexpr int kGemmBN = 256;                    // output columns per tile (MMA N)
constexpr int kGemmStages = 3;                  // weight pipeline depth
constexpr int kAtomBytes = kTile * 128;         // 128 rows x 64 16-bit values
constexpr int kBStageBytes = kGemmBN * 128;     // 256 rows x 64 fp16
constexpr int kStageBytes = kBStageBytes;
constexpr int kGemmThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 norm + epilogue
constexpr int kGemmMaxAtoms = 8;                // R <= 512
constexpr size_t kGemmSmemBytes = (size_t)kGemmMaxAtoms * kAtomBytes + (size_t)kGemmStages * kStageBytes + 1024;

struct GemmParams {
  const __nv_bfloat16* latent;   // [Ttot, R + P]
  const __nv_bfloat16* w_norm;   // [R]
  const int32_t* positions;
  const int32_t* cu;
  const int32_t* tile_seq;
  const int32_t* tile_q0;
  const float* cos_t;
  const float* sin_t;
  __half* k_nope;
  __half* vt;
  __half* k_rot;
  int64_t Ttot;
  int Tpad, R, P, H, N, V, NOUT;
  int tiles_per_cta;             // n tiles (256 columns) per CTA
  int max_pos, interleaved;
  float eps;
  // transposed-value GEMM over cached rows (the eager chunk form): c_hat is
  // already in the padded layout (tile t = rows 128 t ..) and k_rot has been
  // written with it, so the tile's A rows are padded rows and k_rot is left
  int a_padded;
  // 1: k_nope is stored as bf16 (the attention's score operand), 0: as fp16;
  // the buffer holds 16-bit codes
  int knope_bf16;
};

struct GemmBarriers {
  uint64_t a_full, a_ready;
  uint64_t b_full[kGemmStages], b_empty[kGemmStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// grid: (tile capacity, ceil(NOUT / (256 * tiles_per_cta))). The TMA-fed
// prologue normalizes the CTA's 128 x R latent tile in shared memory (fp16,
// resident for all its output tiles); the fp16 weight streams through a
// 3-stage TMA pipeline. The fp32 accumulator is double buffered in TMEM
// (2 x 256 columns) so the epilogue of one output tile overlaps the MMAs of
// the next.
__global__ void __launch_bounds__(kGemmThreads, 1)
norm_kvb_gemm_kernel(const __grid_constant__ CUtensorMap map_lat, const __grid_constant__ CUtensorMap map_w,
                     GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmBarriers bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();         // the schedule and the fp16 weight come from the previous kernel
  pdl_allow_next();
  const int tile = blockIdx.x;
  const int seq = p.tile_seq[tile];
  if (seq < 0) return;   // past the real tiles (uniform over the CTA)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                        // R/64 atoms of [128 x 64]
  uint8_t* sB = smem + kGemmMaxAtoms * kAtomBytes;           // stages of [256 x 64] weight
  const int q0 = p.tile_q0[tile];
  const int64_t seq0 = p.cu[seq];
  const int L = (int)(p.cu[seq + 1] - seq0);
  const int tp0 = tile * kTile;                              // padded row of the tile
  const int natoms = p.R / 64;
  const int n_begin = blockIdx.y * p.tiles_per_cta;
  const int n_tiles_total = (p.NOUT + kGemmBN - 1) / kGemmBN;
  const int n_end = min(n_tiles_total, n_begin + p.tiles_per_cta);
  const int my_tiles = n_end - n_begin;
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.a_full, 1);
    mbar_init(&bars.a_ready, 128);
    for (int s = 0; s < kGemmStages; ++s) { mbar_init(&bars.b_full[s], 1); mbar_init(&bars.b_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&bars.acc_full[s], 1); mbar_init(&bars.acc_empty[s], 128); }
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
    if (lane == 0 && my_tiles > 0) {
      tma_prefetch_desc(&map_lat);
      tma_prefetch_desc(&map_w);
      mbar_arrive_expect_tx(&bars.a_full, natoms * kAtomBytes);
      for (int a = 0; a < natoms; ++a)
        tma_load_2d(sA + a * kAtomBytes, &map_lat, &bars.a_full, a * 64, (int)(seq0 + q0));
      int it = 0;
      bool ok = true;
      for (int nt = n_begin; nt < n_end && ok; ++nt) {
        for (int kc = 0; kc < natoms; ++kc, ++it) {
          const int s = it % kGemmStages;
          const uint32_t ph = (uint32_t)(it / kGemmStages) & 1u;
          if (!mbar_wait(&bars.b_empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* st = sB + s * kStageBytes;
          mbar_arrive_expect_tx(&bars.b_full[s], kStageBytes);
          tma_load_2d(st, &map_w, &bars.b_full[s], kc * 64, nt * kGemmBN);
        }
      }
      if (!ok) {   // drain the loads that may still be in flight before the CTA exits
        mbar_wait_drain(&bars.a_full, 0);
        for (int j = (it > kGemmStages ? it - kGemmStages : 0); j < it; ++j)
          mbar_wait_drain(&bars.b_full[j % kGemmStages], (uint32_t)(j / kGemmStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    if (my_tiles > 0) {
      const uint32_t idesc = idesc_f16_f32(kTile, kGemmBN);
      bool ok = mbar_wait_warp(&bars.a_ready, 0, abort_flag);
      tc_fence_after();
      int it = 0;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int acc = i & 1;
        if (!mbar_wait_warp(&bars.acc_empty[acc], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * kGemmBN);
        for (int kc = 0; kc < natoms; ++kc, ++it) {
          const int s = it % kGemmStages;
          if (!mbar_wait_warp(&bars.b_full[s], (uint32_t)(it / kGemmStages) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc_kmajor_sw128(smem_u32(sA + kc * kAtomBytes));
          const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + s * kStageBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss_elect(d, desc_advance(ad, k * 32), desc_advance(bd, k * 32), idesc, (kc | k) != 0);
          mma_commit_elect(&bars.b_empty[s]);
        }
        if (!ok) break;
        mma_commit_elect(&bars.acc_full[acc]);
      }
      mma_commit_elect(&bars.mma_done);          // every MMA done before TMEM is freed
      if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
      __syncwarp();
    }
  } else {
    // ---------------- RMSNorm prologue, then epilogue (warps 2-5) ----------------
    const int grp = warp & 3;                 // TMEM lane group this warp may access
    const int row = grp * 32 + lane;          // tile row == TMEM lane
    const bool valid = (q0 + row) < L;
    const int64_t t = seq0 + q0 + row;        // token of this row (when valid)
    const int tp = tp0 + row;                 // padded row
    bool ok = my_tiles > 0 ? mbar_wait_warp(&bars.a_full, 0, abort_flag) : false;
    if (ok) {
      // sum of squares of the R latent columns of this row
      float ss = 0.f;
      for (int a = 0; a < natoms; ++a) {
        const uint8_t* base = sA + a * kAtomBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(base + sw128_offset(row, c));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w4[e]);
            ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
          }
        }
      }
      const float r = valid ? 1.0f / sqrtf(ss / (float)p.R + p.eps) : 0.f;
      // c_hat = w * x * r in place, as fp16 (rows past the sequence become zeros)
      for (int a = 0; a < natoms; ++a) {
        uint8_t* base = sA + a * kAtomBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(base + sw128_offset(row, c));
          const uint4 v = *ptr;
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          const int k0 = a * 64 + c * 8;
          const uint4 wv = *reinterpret_cast<const uint4*>(p.w_norm + k0);
          const uint32_t g4[4] = {wv.x, wv.y, wv.z, wv.w};
          uint32_t o4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w4[e]);
            const float2 g = unpack_bf16x2(g4[e]);
            o4[e] = pack_f16x2(g.x * (f.x * r), g.y * (f.y * r));
          }
          *ptr = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
      }
      fence_proxy_async_smem();
    }
    mbar_arrive(&bars.a_ready);
    // rotated shared key of this row (one CTA column per tile writes it)
    if (blockIdx.y == 0) {
      const int half = p.P / 2;
      __half* dst = p.k_rot + (int64_t)tp * p.P;
      if (valid) {
        const __nv_bfloat16* src = p.latent + t * (p.R + p.P) + p.R;
        const int64_t pos = checked_pos(p.positions[t], p.max_pos);
        for (int i = 0; i < half; ++i) {
          int ia, ib;
          rope_pair_slots(i, p.P, p.interleaved, ia, ib);
          float ox, oy;
          rope_turn(__bfloat162float(src[ia]), __bfloat162float(src[ib]), p.cos_t[pos * half + i],
                    p.sin_t[pos * half + i], ox, oy);
          dst[ia] = __float2half_rn(ox);
          dst[ib] = __float2half_rn(oy);
        }
      } else {
        for (int i = 0; i < p.P; ++i) dst[i] = __float2half_rn(0.f);
      }
    }
    // epilogue: TMEM -> k_nope (fp16 or bf16) / transposed values (fp16)
    const int NV = p.N + p.V;
    float vmax = 0.f;
    for (int i = 0; i < my_tiles && ok; ++i) {
      const int acc = i & 1;
      if (!mbar_wait_warp(&bars.acc_full[acc], (uint32_t)(i >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int o_base = (n_begin + i) * kGemmBN;
      for (int ch = 0; ch < kGemmBN / 16; ++ch) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(grp * 32) << 16) + (uint32_t)(acc * kGemmBN + ch * 16), v);
        const int o0 = o_base + ch * 16;
        if (o0 >= p.NOUT) continue;
        const int h = o0 / NV, c0 = o0 % NV;
        if (c0 >= p.N || !p.knope_bf16) {
#pragma unroll
          for (int e = 0; e < 16; ++e) vmax = fmaxf(vmax, fabsf(__uint_as_float(v[e])));
        }
        if (c0 < p.N) {
          uint32_t pk[8];
          if (p.knope_bf16) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pk[e] = pack_f16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
          }
          uint4* dst = reinterpret_cast<uint4*>(p.k_nope + ((int64_t)h * p.Tpad + tp) * p.N + c0);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          __half* dst = p.vt + ((int64_t)h * p.V + (c0 - p.N)) * p.Tpad + tp;
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[(int64_t)e * p.Tpad] = __float2half_rn(__uint_as_float(v[e]));
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[acc]);
    }
    if (!(vmax <= kF16Max)) raise_device_error(kDevErrRange);
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

namespace mla {
namespace tc {

// ---- fused RMSNorm + kv_b_proj GEMM, value half produced transposed --------
// Heads with qk_nope = kN in {64, 128} and v_head = 128. Per head h and
// 128-token tile, two tensor-core products share the resident normalized
// latent tile c_hat [128 x R] (fp16, written by prefill_prep_kernel in token
// order: the rows of a sequence's last tile past its end belong to the next
// sequence, so their outputs are finite, and attention gives those keys zero
// weight) and one streamed weight stage (the head's kN + 128 rows of W, 64 K
// columns per stage):
//   D1 = c_hat W_K^T   M = 128 tokens,   N = kN      -> k_nope rows
//   D2 = W_V c_hat^T   M = 128 channels, N = 128 tokens -> value rows of vt
// The products are the same sums as one c_hat [W_K; W_V]^T; swapping the
// operands of the value half puts one value channel in each TMEM lane, so
// the epilogue writes every transposed value row as 256 contiguous bytes.
// Warps: 0 TMA, 1 MMA, 2-5 the k_nope epilogue, 6-9 the rotated shared key,
// then the value epilogue.
constexpr int kG2Threads = 320;
constexpr int kG2Stages = 3;
constexpr int kG2StageBytes = 256 * 128;
constexpr size_t kG2SmemBytes = (size_t)kGemmMaxAtoms * kAtomBytes + (size_t)kG2Stages * kG2StageBytes + 1024;

template <int kN>
__global__ void __launch_bounds__(kG2Threads, 1)
norm_kvb_gemm_vt_kernel(const __grid_constant__ CUtensorMap map_chat, const __grid_constant__ CUtensorMap map_w,
                        GemmParams p) {
  constexpr int kV = 128;
  constexpr int kRows = kN + kV;                  // weight rows of one head
  constexpr int kStage = kRows * 128;             // bytes of one stage
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ GemmBarriers bars;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();         // the schedule, the fp16 weight and c_hat come from the previous kernel
  pdl_allow_next();
  const int tile = blockIdx.x;
  const int seq = p.tile_seq[tile];
  if (seq < 0) return;   // past the real tiles (uniform over the CTA)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGemmMaxAtoms * kAtomBytes;
  const int q0 = p.tile_q0[tile];
  const int64_t seq0 = p.cu[seq];
  const int L = (int)(p.cu[seq + 1] - seq0);
  const int tp0 = tile * kTile;
  const int natoms = p.R / 64;
  const int h_begin = blockIdx.y * p.tiles_per_cta;
  const int h_end = min(p.H, h_begin + p.tiles_per_cta);
  const int my_heads = h_end - h_begin;
  volatile int* abort_flag = &bars.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&bars.a_full, 1);
    mbar_init(&bars.a_ready, 128);
    for (int s = 0; s < kG2Stages; ++s) { mbar_init(&bars.b_full[s], 1); mbar_init(&bars.b_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&bars.acc_full[s], 1); mbar_init(&bars.acc_empty[s], 256); }
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
    if (lane == 0 && my_heads > 0) {
      tma_prefetch_desc(&map_chat);
      tma_prefetch_desc(&map_w);
      mbar_arrive_expect_tx(&bars.a_full, natoms * kAtomBytes);
      const int arow = p.a_padded ? tp0 : (int)(seq0 + q0);
      for (int a = 0; a < natoms; ++a)
        tma_load_2d(sA + a * kAtomBytes, &map_chat, &bars.a_full, a * 64, arow);
      int it = 0;
      bool ok = true;
      for (int h = h_begin; h < h_end && ok; ++h) {
        for (int kc = 0; kc < natoms; ++kc, ++it) {
          const int s = it % kG2Stages;
          if (!mbar_wait(&bars.b_empty[s], ((uint32_t)(it / kG2Stages) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.b_full[s], kStage);
          tma_load_2d(sB + s * kG2StageBytes, &map_w, &bars.b_full[s], kc * 64, h * kRows);
        }
      }
      if (!ok) {
        mbar_wait_drain(&bars.a_full, 0);
        for (int j = (it > kG2Stages ? it - kG2Stages : 0); j < it; ++j)
          mbar_wait_drain(&bars.b_full[j % kG2Stages], (uint32_t)(j / kG2Stages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
    if (my_heads > 0) {
      const uint32_t idesc1 = idesc_f16_f32(kTile, kN);
      const uint32_t idesc2 = idesc_f16_f32(kTile, kTile);
      bool ok = mbar_wait_warp(&bars.a_ready, 0, abort_flag);
      tc_fence_after();
      int it = 0;
      for (int i = 0; i < my_heads && ok; ++i) {
        const int acc = i & 1;
        if (!mbar_wait_warp(&bars.acc_empty[acc], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d1 = tmem + (uint32_t)(acc * 256);
        const uint32_t d2 = d1 + (uint32_t)kN;
        for (int kc = 0; kc < natoms; ++kc, ++it) {
          const int s = it % kG2Stages;
          if (!mbar_wait_warp(&bars.b_full[s], (uint32_t)(it / kG2Stages) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t cd = desc_kmajor_sw128(smem_u32(sA + kc * kAtomBytes));
          const uint64_t wk = desc_kmajor_sw128(smem_u32(sB + s * kG2StageBytes));
          const uint64_t wv = desc_kmajor_sw128(smem_u32(sB + s * kG2StageBytes + kN * 128));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            mma_ss_elect(d1, desc_advance(cd, k * 32), desc_advance(wk, k * 32), idesc1, (kc | k) != 0);
            mma_ss_elect(d2, desc_advance(wv, k * 32), desc_advance(cd, k * 32), idesc2, (kc | k) != 0);
          }
          mma_commit_elect(&bars.b_empty[s]);
        }
        if (!ok) break;
        mma_commit_elect(&bars.acc_full[acc]);
      }
      mma_commit_elect(&bars.mma_done);
      if (lane == 0) mbar_wait_drain(&bars.mma_done, 0);
      __syncwarp();
    }
  } else {
    const int half = (warp - 2) >> 2;          // 0: norm + k_nope, 1: k_rot + values
    const int grp = warp & 3;
    const int lrow = grp * 32 + lane;          // TMEM lane of this thread
    const uint32_t lane_base = (uint32_t)(grp * 32) << 16;
    bool ok = my_heads > 0;
    if (half == 0) {
      // c_hat arrives in fp16 from the preparation kernel: nothing to do
      // before the epilogue but pass the tile on
      if (ok) ok = mbar_wait_warp(&bars.a_full, 0, abort_flag);
      mbar_arrive(&bars.a_ready);
    } else if (blockIdx.y == 0 && !p.a_padded) {
      // rotated shared key of token row lrow (one CTA column per tile writes
      // it); P = 64: the row's 64 values and its 32 cos / sin entries come in
      // as independent vector loads
      const bool valid = (q0 + lrow) < L;
      const int64_t t = seq0 + q0 + lrow;
      uint4* dst = reinterpret_cast<uint4*>(p.k_rot + (int64_t)(tp0 + lrow) * 64);
      if (valid) {
        const uint4* src = reinterpret_cast<const uint4*>(p.latent + t * (p.R + 64) + p.R);
        const int64_t pos = checked_pos(p.positions[t], p.max_pos);
        const float4* c4 = reinterpret_cast<const float4*>(p.cos_t + pos * 32);
        const float4* s4 = reinterpret_cast<const float4*>(p.sin_t + pos * 32);
        uint4 raw[8];
        float4 cv[8], sv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) { raw[i] = src[i]; cv[i] = c4[i]; sv[i] = s4[i]; }
        float x[64], y[64], cs[32], sn[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w4[e]);
            x[i * 8 + 2 * e] = f.x;
            x[i * 8 + 2 * e + 1] = f.y;
          }
          cs[4 * i] = cv[i].x; cs[4 * i + 1] = cv[i].y; cs[4 * i + 2] = cv[i].z; cs[4 * i + 3] = cv[i].w;
          sn[4 * i] = sv[i].x; sn[4 * i + 1] = sv[i].y; sn[4 * i + 2] = sv[i].z; sn[4 * i + 3] = sv[i].w;
        }
        if (p.interleaved) {
#pragma unroll
          for (int i = 0; i < 32; ++i) rope_turn(x[2 * i], x[2 * i + 1], cs[i], sn[i], y[2 * i], y[2 * i + 1]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) rope_turn(x[i], x[i + 32], cs[i], sn[i], y[i], y[i + 32]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_uint4(pack_f16x2(y[8 * i], y[8 * i + 1]), pack_f16x2(y[8 * i + 2], y[8 * i + 3]),
                              pack_f16x2(y[8 * i + 4], y[8 * i + 5]), pack_f16x2(y[8 * i + 6], y[8 * i + 7]));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // epilogue: half 0 writes k_nope rows (lane = token), half 1 value rows (lane = channel)
    float vmax = 0.f;
    for (int i = 0; i < my_heads && ok; ++i) {
      const int acc = i & 1;
      const int h = h_begin + i;
      if (!mbar_wait_warp(&bars.acc_full[acc], (uint32_t)(i >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t src = tmem + lane_base + (uint32_t)(acc * 256 + (half ? kN : 0));
      uint4* dst = half ? reinterpret_cast<uint4*>(p.vt + ((int64_t)h * kV + lrow) * p.Tpad + tp0)
                        : reinterpret_cast<uint4*>(p.k_nope + ((int64_t)h * p.Tpad + tp0 + lrow) * kN);
      const int nchunks = half ? kTile / 32 : kN / 32;
      const bool kb = !half && p.knope_bf16;   // warp-uniform
      for (int c = 0; c < nchunks; ++c) {
        uint32_t v[32];
        tmem_ld32(src + (uint32_t)(c * 32), v);
        uint32_t pk[16];
        if (kb) {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = __uint_as_float(v[2 * e]), b = __uint_as_float(v[2 * e + 1]);
            vmax = fmaxf(vmax, fmaxf(fabsf(a), fabsf(b)));
            pk[e] = pack_f16x2(a, b);
          }
        }
        st_global_v8(dst + c * 4, pk);
        st_global_v8(dst + c * 4 + 2, pk + 8);
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[acc]);
    }
    if (!(vmax <= kF16Max)) raise_device_error(kDevErrRange);
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
