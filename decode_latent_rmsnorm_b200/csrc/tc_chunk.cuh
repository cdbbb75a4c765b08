// Chunks of new tokens that continue cached sequences, eager form: the keys
// and values of every row of each sequence (its cached prefix and the chunk
// just appended) are expanded by the up-projection GEMM, and the chunk's
// queries attend to them with the two-tile attention kernel, causally in
// absolute positions.
//
// Source: GLM-5 "Normalized key-value latent" page, "KV cache": the cache is
// updated with the new tokens' normalized latent and rotated key first, and
// the heads are then expanded from every cached row; Kimi-K2 "Query content
// heads" page, "Join query parts": the attention of a multi-token query.
//
// For sequence s with p = prefix_lens[s] cached rows and n chunk tokens, the
// keys are its Lk = p + n cache rows (rows cache_offsets[s] .. + Lk - 1); chunk
// token i is query i with key offset p (it attends keys 0 .. p + i). The keys
// sit in a padded layout like the prefill's: every sequence's first key on a
// 128-row boundary, rows past Lk zero.
#pragma once
#include "tc_gemm.cuh"

namespace mla {
namespace tc {

// Validity of sequence s: consistent bounds, a prefix inside the cache, the
// whole sequence within max_total_len and the rotary table.
__device__ __forceinline__ bool chunk_seq_ok(const int32_t* cu, int s, int64_t n_tokens,
                                             const int64_t* cache_offsets, const int32_t* prefix_lens,
                                             int max_total_len, int max_pos, int64_t cache_num_rows) {
  const int64_t a = cu[s], b = cu[s + 1], p = prefix_lens[s], o = cache_offsets[s];
  return a >= 0 && b >= a && b <= n_tokens && p >= 0 && o >= 0 && p + (b - a) <= (int64_t)max_total_len &&
         o + p + (b - a) <= cache_num_rows && p + (b - a) <= (int64_t)max_pos;
}

// Schedule of the eager form, run by one block of 1024 threads:
//   seq_ok[s]                      1 for a valid sequence, else 0 (no tiles,
//                                  no blocks; the device error word is set)
//   kseq_tile0[s]                  first padded key tile of sequence s
//   ktile_seq[t], ktile_k0[t]      sequence and first key row of key tile t
//   qblk_seq[j], qblk_q0[j]        the 256-row query blocks, sorted by
//                                  decreasing causal work (keys before the
//                                  block's last row); qorder[j] = j
// Entries past the real tiles / blocks are -1; *item_counter = 0 (the
// attention's work counter).
constexpr int kChunkSchedThreads = 1024;
__global__ void __launch_bounds__(kChunkSchedThreads)
chunk_eager_schedule_kernel(const int32_t* __restrict__ cu, int nseq, int64_t n_tokens,
                            const int64_t* __restrict__ cache_offsets, const int32_t* __restrict__ prefix_lens,
                            int max_total_len, int max_pos, int64_t cache_num_rows, int kcap, int qcap,
                            int32_t* __restrict__ seq_ok, int32_t* __restrict__ kseq_tile0,
                            int32_t* __restrict__ ktile_seq, int32_t* __restrict__ ktile_k0,
                            int32_t* __restrict__ qblk_seq, int32_t* __restrict__ qblk_q0,
                            int32_t* __restrict__ qorder, int32_t* __restrict__ item_counter) {
  constexpr int kBuckets = 2048;
  __shared__ int s_scan[1024];
  __shared__ int s_carry, s_overflow;
  __shared__ int s_cnt[kBuckets];
  __shared__ int s_off[kBuckets];
  const int tid = threadIdx.x;
  if (tid == 0) { s_carry = 0; s_overflow = 0; *item_counter = 0; }
  for (int i = tid; i < kcap; i += blockDim.x) { ktile_seq[i] = -1; ktile_k0[i] = -1; }
  for (int i = tid; i < qcap; i += blockDim.x) { qblk_seq[i] = -1; qblk_q0[i] = -1; qorder[i] = -1; }
  for (int k = tid; k < kBuckets; k += blockDim.x) { s_cnt[k] = 0; s_off[k] = 0; }
  __syncthreads();
  // 1) validity, key tiles per sequence -> exclusive scan into kseq_tile0;
  //    query-block counts per work bucket
  for (int base = 0; base <= nseq; base += blockDim.x) {
    const int s = base + tid;
    int nt = 0;
    if (s < nseq) {
      const bool ok = chunk_seq_ok(cu, s, n_tokens, cache_offsets, prefix_lens, max_total_len, max_pos,
                                   cache_num_rows);
      seq_ok[s] = ok ? 1 : 0;
      if (!ok) {
        raise_device_error(kDevErrBadInput);
      } else {
        const int n = cu[s + 1] - cu[s], p = prefix_lens[s];
        nt = (p + n + kTile - 1) / kTile;
        for (int q0 = 0; q0 < n; q0 += 2 * kTile) {
          const int last = min(q0 + 2 * kTile, n) - 1;
          atomicAdd(&s_cnt[min((p + last) / (2 * kTile), kBuckets - 1)], 1);
        }
      }
    }
    const int inc = block_inclusive_scan_1024(nt, s_scan);
    if (s <= nseq) kseq_tile0[s] = s_carry + inc - nt;
    __syncthreads();
    if (tid == (int)blockDim.x - 1) s_carry += inc;
    __syncthreads();
  }
  if (s_carry > kcap) {   // cannot happen for valid input (the host bounds kcap); guards the arrays
    if (tid == 0) raise_device_error(kDevErrBadInput);
    return;
  }
  // 2) key tiles
  for (int s = tid; s < nseq; s += blockDim.x) {
    const int t0 = kseq_tile0[s], nt = kseq_tile0[s + 1] - t0;
    for (int k = 0; k < nt; ++k) { ktile_seq[t0 + k] = s; ktile_k0[t0 + k] = k * kTile; }
  }
  // 3) query blocks in decreasing work order (descending exclusive offsets of
  //    the buckets; thread i owns reversed buckets 2i and 2i + 1)
  {
    const int k0 = kBuckets - 1 - 2 * tid, k1 = k0 - 1;
    const int c0 = s_cnt[k0], c1 = s_cnt[k1];
    const int before = block_inclusive_scan_1024(c0 + c1, s_scan) - (c0 + c1);
    s_off[k0] = before;
    s_off[k1] = before + c0;
  }
  __syncthreads();
  for (int s = tid; s < nseq; s += blockDim.x) {
    if (!seq_ok[s]) continue;
    const int n = cu[s + 1] - cu[s], p = prefix_lens[s];
    for (int q0 = 0; q0 < n; q0 += 2 * kTile) {
      const int last = min(q0 + 2 * kTile, n) - 1;
      const int pos = atomicAdd(&s_off[min((p + last) / (2 * kTile), kBuckets - 1)], 1);
      if (pos < qcap) { qblk_seq[pos] = s; qblk_q0[pos] = q0; qorder[pos] = pos; }
      else s_overflow = 1;
    }
  }
  __syncthreads();
  if (tid == 0 && s_overflow) raise_device_error(kDevErrBadInput);
}

// The padded key rows: one warp per row tp < n_rows. Row k of sequence s's
// keys is cache row cache_offsets[s] + k: its normalized latent goes to c16
// [tp, :R] and its rotated key to k_rot [tp, :64], both fp16 (exact for values
// in fp16's normal range; a value beyond the fp16 range sets the device error
// word); rows past the sequence's keys are zero. R <= 512, P = 64.
constexpr int kChunkRowsPerBlock = 8;
__global__ void __launch_bounds__(32 * kChunkRowsPerBlock)
chunk_eager_rows_kernel(const __nv_bfloat16* __restrict__ cache, int R, const int64_t* __restrict__ cache_offsets,
                        const int32_t* __restrict__ prefix_lens, const int32_t* __restrict__ cu,
                        const int32_t* __restrict__ ktile_seq, const int32_t* __restrict__ ktile_k0,
                        int64_t n_rows, __half* __restrict__ c16, __half* __restrict__ k_rot) {
  pdl_wait();         // the schedule and the appended chunk rows come from the previous kernels
  pdl_allow_next();
  const int64_t tp = (int64_t)blockIdx.x * kChunkRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tp >= n_rows) return;
  const int s = ktile_seq[tp / kTile];
  if (s < 0) return;                        // past the real tiles: never read
  const int k = ktile_k0[tp / kTile] + (int)(tp % kTile);
  const int Lk = prefix_lens[s] + (cu[s + 1] - cu[s]);
  const int nch = R / 8;                    // 16-byte chunks of the latent
  uint4* dst = reinterpret_cast<uint4*>(c16 + tp * R);
  uint2* dr = reinterpret_cast<uint2*>(k_rot + tp * 64);   // 4 values per lane
  if (k >= Lk) {
    for (int c = lane; c < nch; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    dr[lane & 15] = make_uint2(0u, 0u);
    return;
  }
  const __nv_bfloat16* src = cache + (cache_offsets[s] + k) * (int64_t)(R + 64);
  float mx = 0.f;
  for (int c = lane; c < nch; c += 32) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[c];
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t o4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w4[e]);
      mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
      o4[e] = pack_f16x2(f.x, f.y);
    }
    dst[c] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
  if (lane < 16) {
    const uint2 v = reinterpret_cast<const uint2*>(src + R)[lane];
    const float2 f0 = unpack_bf16x2(v.x), f1 = unpack_bf16x2(v.y);
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
    dr[lane] = make_uint2(pack_f16x2(f0.x, f0.y), pack_f16x2(f1.x, f1.y));
  }
  if (!(mx <= kF16Max)) raise_device_error(kDevErrRange);
}

// Output rows of the chunk tokens of invalid sequences are zero (as in the
// absorbed form). One warp per chunk token; the sequence is found by a
// bounded binary search (it ends after log2(nseq) + 1 steps even when
// cu_seqlens is not sorted).
__global__ void __launch_bounds__(32 * kChunkRowsPerBlock)
chunk_eager_zero_kernel(const int32_t* __restrict__ cu, int nseq, int64_t n_tokens,
                        const int32_t* __restrict__ seq_ok, int HV, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_allow_next();
  const int64_t t = (int64_t)blockIdx.x * kChunkRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= n_tokens) return;
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)cu[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const bool inside = (int64_t)cu[lo] <= t && t < (int64_t)cu[lo + 1];
  if (inside && seq_ok[lo]) return;
  uint4* o = reinterpret_cast<uint4*>(out + t * HV);
  for (int c = lane; c < HV / 8; c += 32) o[c] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace tc
}  // namespace mla
