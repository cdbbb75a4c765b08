// Chunks of new tokens that continue cached sequences: per-token bookkeeping.
//
// Source: GLM-5 "Normalized key-value latent" page, "KV cache". The cache is
// updated with the new tokens' normalized latent and rotated key first, and
// the heads are then expanded from every cached row. A chunk token therefore
// sees its sequence's cached prefix, the chunk tokens before it, and itself.
//
// For chunk token t of sequence s (cu_seqlens[s] <= t < cu_seqlens[s + 1]),
// with p = prefix_lens[s], o = cache_offsets[s] and i = t - cu_seqlens[s]:
//   position      p + i             (rotary position of its key and query)
//   cache row     o + p + i         (where its normalized latent goes)
//   attended rows o .. o + p + i    (offset o, length p + i + 1)
// The append kernel consumes (position, cache row); the absorbed decode
// consumes (position, offset, length), one decode row per chunk token.
#pragma once
#include "common.cuh"

namespace mla {

constexpr int kChunkThreads = 256;

// One thread per chunk token. A token whose sequence cannot be found, or
// whose rows or position fall outside their ranges, gets cache row -1 and
// length 0 (the append and the decode both skip such a token; its output is
// zero) and sets the device error word.
__global__ void __launch_bounds__(kChunkThreads)
chunk_rows_kernel(const int32_t* __restrict__ cu_seqlens, int nseq, int64_t n_tokens,
                  const int64_t* __restrict__ cache_offsets, const int32_t* __restrict__ prefix_lens,
                  int max_total_len, int max_pos, int64_t cache_num_rows, int32_t* __restrict__ positions,
                  int64_t* __restrict__ cache_rows, int64_t* __restrict__ attend_offsets,
                  int32_t* __restrict__ attend_lens) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_tokens) return;
  if (t == 0 && (cu_seqlens[0] != 0 || (int64_t)cu_seqlens[nseq] != n_tokens)) raise_device_error(kDevErrBadInput);
  // the last sequence s in [0, nseq) with cu_seqlens[s] <= t (the interval
  // shrinks every step, so this ends after at most log2(nseq) + 1 steps
  // even when cu_seqlens is not sorted)
  int lo = 0, hi = nseq - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)cu_seqlens[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int64_t a = cu_seqlens[lo], b = cu_seqlens[lo + 1];
  const int64_t p = prefix_lens[lo], o = cache_offsets[lo];
  const int64_t i = t - a, n = b - a;
  const bool ok = a <= t && t < b && p >= 0 && o >= 0 && p + n <= (int64_t)max_total_len &&
                  o + p + n <= cache_num_rows && p + i < (int64_t)max_pos;
  if (!ok) raise_device_error(kDevErrBadInput);
  positions[t] = ok ? (int32_t)(p + i) : 0;
  cache_rows[t] = ok ? o + p + i : -1;
  attend_offsets[t] = ok ? o : 0;
  attend_lens[t] = ok ? (int32_t)(p + i + 1) : 0;
}

}  // namespace mla
