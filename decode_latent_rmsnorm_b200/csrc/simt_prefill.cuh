// CUDA-core (FFMA) prefill kernels: exact fp32 arithmetic for MLA_FP32 runs
// and for head geometries the tensor-core kernels do not take.
//
// Sources: "Eager latent expansion" equation page (latent split,
// kv_a_layernorm, kv_b_proj, view per head, split into k_nope / value);
// Kimi-K2 "RoPE coefficients" page, "Key heads" (mla-kv, mla-prefill) and
// Kimi-K2 "Query content heads" page, "Join query parts" (rotation, joined
// query/key, scaled scores, causal mask, fp32 softmax, P @ V).
#pragma once
#include "common.cuh"

namespace mla {
namespace simt {

constexpr int kGemmBM = 64, kGemmBN = 64, kGemmBK = 16;

// kv[t, o] = sum_k c_hat[t, k] W[o, k] with c_hat = w * c / sqrt(mean(c^2) + eps),
// scattered into k_nope [H, Ttot, N] and values [H, Ttot, V] (head-major).
// The RMS factor of each of the tile's rows is computed in the prologue from
// the latent row itself, so the normalized latent never touches memory.
template <typename T>
__global__ void __launch_bounds__(256)
norm_proj_kernel(const T* __restrict__ latent, const T* __restrict__ W,
                 const T* __restrict__ w_norm, int64_t Ttot, int R, int P, int H, int N, int V,
                 float eps, T* __restrict__ k_nope, T* __restrict__ vals) {
  __shared__ float rfac[kGemmBM];
  __shared__ float As[kGemmBK][kGemmBM + 4];
  __shared__ float Bs[kGemmBK][kGemmBN + 4];
  const int tid = threadIdx.x;
  const int64_t m0 = (int64_t)blockIdx.x * kGemmBM;
  const int n0 = blockIdx.y * kGemmBN;
  const int NOUT = H * (N + V);
  const int ld = R + P;

  // Prologue: one warp per 8 rows, mean square over the R latent columns.
  const int warp = tid >> 5, lane = tid & 31;
  for (int r = warp; r < kGemmBM; r += 8) {
    const int64_t t = m0 + r;
    float ss = 0.f;
    if (t < Ttot)
      for (int k = lane; k < R; k += 32) {
        const float x = to_f32(latent[t * ld + k]);
        ss += x * x;
      }
    ss = warp_sum(ss);
    if (lane == 0) rfac[r] = 1.0f / sqrtf(ss / (float)R + eps);
  }
  __syncthreads();

  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < R; k0 += kGemmBK) {
    for (int e = tid; e < kGemmBM * kGemmBK; e += 256) {
      const int r = e / kGemmBK, k = e % kGemmBK;
      const int64_t t = m0 + r;
      float v = 0.f;
      if (t < Ttot) v = to_f32(latent[t * ld + k0 + k]) * to_f32(w_norm[k0 + k]) * rfac[r];
      As[k][r] = v;
    }
    for (int e = tid; e < kGemmBN * kGemmBK; e += 256) {
      const int n = e / kGemmBK, k = e % kGemmBK;
      const int o = n0 + n;
      Bs[k][n] = (o < NOUT) ? to_f32(W[(int64_t)o * R + k0 + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kGemmBK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t t = m0 + ty * 4 + i;
    if (t >= Ttot) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = n0 + tx * 4 + j;
      if (o >= NOUT) continue;
      const int h = o / (N + V), c = o % (N + V);
      if (c < N) k_nope[((int64_t)h * Ttot + t) * N + c] = from_f32<T>(acc[i][j]);
      else vals[((int64_t)h * Ttot + t) * V + (c - N)] = from_f32<T>(acc[i][j]);
    }
  }
}

// The one rotary key per token, rotated at its position: k_rot [Ttot, P].
template <typename T>
__global__ void rope_key_kernel(const T* __restrict__ latent, const int32_t* __restrict__ positions,
                                const float* __restrict__ cos_t, const float* __restrict__ sin_t,
                                int max_pos, int64_t Ttot, int R, int P, int interleaved,
                                T* __restrict__ k_rot) {
  const int half = P / 2;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= Ttot * half) return;
  const int64_t t = idx / half;
  const int i = (int)(idx % half);
  int a, b;
  rope_pair_slots(i, P, interleaved, a, b);
  const int64_t pos = checked_pos(positions[t], max_pos);
  const float c = cos_t[pos * half + i], s = sin_t[pos * half + i];
  const T* src = latent + t * (R + P) + R;
  float ox, oy;
  rope_turn(to_f32(src[a]), to_f32(src[b]), c, s, ox, oy);
  k_rot[t * P + a] = from_f32<T>(ox);
  k_rot[t * P + b] = from_f32<T>(oy);
}

constexpr int kAttBQ = 32, kAttBKV = 32, kAttMaxVPerThread = 32;

// Causal attention for one (query block, sequence, head). 256 threads: each
// query row is owned by 8 consecutive lanes; scores are kept online (running
// max and sum), so the [L, L] matrix is never formed.
// kPadded = false: k_nope [H, Ttot, N], vals [H, Ttot, V], k_rot [Ttot, P];
// kPadded = true: the tensor-core GEMM's padded layout, k_nope [H, Tpad, N],
// vals transposed [H, V, Tpad], k_rot [Tpad, P], sequence s starting at
// padded row 128 * seq_tile0[s].
template <typename T, bool kPadded>
__global__ void __launch_bounds__(256)
attention_kernel(const T* __restrict__ q, const T* __restrict__ k_nope, const T* __restrict__ k_rot,
                 const T* __restrict__ vals, const int32_t* __restrict__ positions,
                 const int32_t* __restrict__ cu_seqlens, const float* __restrict__ cos_t,
                 const float* __restrict__ sin_t, int max_pos, int max_seqlen, int64_t Ttot, int H,
                 int N, int P, int V, int interleaved, float scale, T* __restrict__ out,
                 const int32_t* __restrict__ seq_tile0, int64_t Tpad) {
  extern __shared__ float smem[];
  const int D = N + P;
  float* Qs = smem;                       // [BQ][D]
  float* Ks = Qs + kAttBQ * D;            // [BKV][D]
  float* Vs = Ks + kAttBKV * D;           // [BKV][V]
  float* Ps = Vs + kAttBKV * V;           // [BQ][BKV]
  const int s = blockIdx.y, h = blockIdx.z;
  const int tid = threadIdx.x;
  const int64_t seq0 = cu_seqlens[s], seq1 = cu_seqlens[s + 1];
  if (seq0 < 0 || seq1 < seq0 || seq1 > Ttot || seq1 - seq0 > max_seqlen) {   // bad boundaries
    if (blockIdx.x == 0 && h == 0 && tid == 0) raise_device_error(kDevErrBadInput);
    return;
  }
  const int L = (int)(seq1 - seq0);
  const int q0 = blockIdx.x * kAttBQ;
  if (q0 >= L) return;
  const int half = P / 2;
  const int64_t kv0 = kPadded ? (int64_t)seq_tile0[s] * 128 : seq0;   // row of key 0 in the K/V buffers
  const int64_t kv_rows = kPadded ? Tpad : Ttot;

  for (int e = tid; e < kAttBQ * D; e += 256) {
    const int r = e / D, d = e % D;
    float v = 0.f;
    if (q0 + r < L) {
      const int64_t t = seq0 + q0 + r;
      const T* qr = q + (t * H + h) * D;
      if (d < N) {
        v = to_f32(qr[d]);
      } else {
        const int j = d - N;
        const int i = interleaved ? (j >> 1) : (j % half);
        int a, b;
        rope_pair_slots(i, P, interleaved, a, b);
        const int64_t pos = checked_pos(positions[t], max_pos);
        float ox, oy;
        rope_turn(to_f32(qr[N + a]), to_f32(qr[N + b]), cos_t[pos * half + i], sin_t[pos * half + i],
                  ox, oy);
        v = (j == a) ? ox : oy;
      }
    }
    Qs[e] = v;
  }

  const int row = tid >> 3, sub = tid & 7;
  const bool row_valid = (q0 + row) < L;
  float m = -INFINITY, l = 0.f;
  float acc[kAttMaxVPerThread];
#pragma unroll
  for (int c = 0; c < kAttMaxVPerThread; ++c) acc[c] = 0.f;
  const int nv = V / 8;
  const int kv_end = min(L, q0 + kAttBQ);

  for (int k0 = 0; k0 < kv_end; k0 += kAttBKV) {
    __syncthreads();
    for (int e = tid; e < kAttBKV * D; e += 256) {
      const int r = e / D, d = e % D;
      float v = 0.f;
      if (k0 + r < L) {
        const int64_t t = kv0 + k0 + r;
        v = d < N ? to_f32(k_nope[((int64_t)h * kv_rows + t) * N + d]) : to_f32(k_rot[t * P + (d - N)]);
      }
      Ks[e] = v;
    }
    for (int e = tid; e < kAttBKV * V; e += 256) {
      const int r = e / V, d = e % V;
      const int64_t t = kv0 + k0 + r;
      float v = 0.f;
      if (k0 + r < L)
        v = kPadded ? to_f32(vals[((int64_t)h * V + d) * kv_rows + t]) : to_f32(vals[((int64_t)h * kv_rows + t) * V + d]);
      Vs[e] = v;
    }
    __syncthreads();
    float sc[kAttBKV / 8];
    float tmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < kAttBKV / 8; ++c) {
      const int col = sub + 8 * c;
      float d = 0.f;
      for (int x = 0; x < D; ++x) d = fmaf(Qs[row * D + x], Ks[col * D + x], d);
      d *= scale;
      if (k0 + col > q0 + row || k0 + col >= L) d = -INFINITY;   // causal mask
      sc[c] = d;
      tmax = fmaxf(tmax, d);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float m_new = fmaxf(m, tmax);
    float alpha = 1.f, psum = 0.f;
    if (row_valid) {
      alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
#pragma unroll
      for (int c = 0; c < kAttBKV / 8; ++c) {
        const float p = (sc[c] == -INFINITY) ? 0.f : expf(sc[c] - m_new);
        Ps[row * kAttBKV + sub + 8 * c] = p;
        psum += p;
      }
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    __syncthreads();
    if (row_valid) {
      m = m_new;
      l = l * alpha + psum;
      for (int c = 0; c < nv; ++c) {
        float a = acc[c] * alpha;
        const int col = sub + 8 * c;
        for (int j = 0; j < kAttBKV; ++j) a = fmaf(Ps[row * kAttBKV + j], Vs[j * V + col], a);
        acc[c] = a;
      }
    }
  }
  if (row_valid) {
    const int64_t t = seq0 + q0 + row;
    const float inv = 1.f / l;
    for (int c = 0; c < nv; ++c) out[(t * H + h) * V + sub + 8 * c] = from_f32<T>(acc[c] * inv);
  }
}

inline size_t attention_smem_bytes(int D, int V) {
  return sizeof(float) * ((size_t)kAttBQ * D + (size_t)kAttBKV * D + (size_t)kAttBKV * V +
                          (size_t)kAttBQ * kAttBKV);
}

// New cache rows: RMSNorm of the latent and the rotated key, one block per row.
template <typename T>
__global__ void __launch_bounds__(256)
cache_append_kernel(const T* __restrict__ latent, const T* __restrict__ w_norm,
                    const int32_t* __restrict__ positions, const float* __restrict__ cos_t,
                    const float* __restrict__ sin_t, int max_pos, int R, int P, int interleaved,
                    float eps, T* __restrict__ cache, int64_t cache_num_rows,
                    const int64_t* __restrict__ cache_rows) {
  __shared__ float red[8];
  const int64_t i = blockIdx.x;
  const T* src = latent + i * (R + P);
  const int64_t row = cache_rows[i];
  const int64_t pos_raw = positions[i];
  if (row < 0 || row >= cache_num_rows || pos_raw < 0 || pos_raw >= max_pos) {
    if (threadIdx.x == 0) raise_device_error(kDevErrBadInput);
    return;
  }
  T* dst = cache + row * (R + P);
  float ss = 0.f;
  for (int k = threadIdx.x; k < R; k += blockDim.x) {
    const float x = to_f32(src[k]);
    ss += x * x;
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
  const float r = 1.0f / sqrtf(tot / (float)R + eps);
  for (int k = threadIdx.x; k < R; k += blockDim.x)
    dst[k] = from_f32<T>(to_f32(w_norm[k]) * (to_f32(src[k]) * r));
  const int half = P / 2;
  const int64_t pos = pos_raw;
  for (int p = threadIdx.x; p < half; p += blockDim.x) {
    int a, b;
    rope_pair_slots(p, P, interleaved, a, b);
    float ox, oy;
    rope_turn(to_f32(src[R + a]), to_f32(src[R + b]), cos_t[pos * half + p], sin_t[pos * half + p],
              ox, oy);
    dst[R + a] = from_f32<T>(ox);
    dst[R + b] = from_f32<T>(oy);
  }
}

}  // namespace simt
}  // namespace mla
