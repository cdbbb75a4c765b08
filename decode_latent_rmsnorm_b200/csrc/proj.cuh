// The projections on either side of the path: kv_a_proj_with_mqa (hidden ->
// compressed_kv), q_a_proj -> q_a_layernorm -> q_b_proj (hidden -> q) and
// o_proj (attention output -> hidden).
//
// Source: Kimi-K2 "RoPE coefficients" page, "Query heads" (mla-init: the
// nn.Linear shapes and the query RMSNorm; mla-queries: their order) and "Key
// heads" (mla-kv: the joint down-projection feeding the latent RMSNorm).
//
// A Linear is out[t, j] = sum_k x[t, k] w[j, k] (w the nn.Linear weight
// [out, in]). In bf16 with K a multiple of 64 it runs on the tensor cores
// (head_gemm_kernel with one head); these kernels are the rest: the query
// RMSNorm, and a CUDA-core Linear for fp32 runs and other K.
#pragma once
#include "tc_ptx.cuh"

namespace mla {

constexpr int kRowsPerNormBlock = 8;   // one warp per row

// y[t, :] = w * x[t, :] / sqrt(mean(x[t, :]^2) + eps) over `width` values,
// fp32 arithmetic. x and y may be the same buffer: each lane reads the values
// it writes before writing them.
template <typename T>
__global__ void __launch_bounds__(32 * kRowsPerNormBlock)
rmsnorm_rows_kernel(const T* x, const T* __restrict__ w, T* y, int64_t rows, int width, float eps) {
  const int64_t t = (int64_t)blockIdx.x * kRowsPerNormBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= rows) return;
  const T* xr = x + t * width;
  float ss = 0.f;
  for (int k = lane; k < width; k += 32) {
    const float v = to_f32(xr[k]);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)width + eps);
  T* yr = y + t * width;
  for (int k = lane; k < width; k += 32) yr[k] = from_f32<T>(to_f32(w[k]) * (to_f32(xr[k]) * r));
}

// The query RMSNorm of a bf16 run, on q_a_proj's fp32 result (never rounded
// before the norm): y[t, :] = w * x[t, :] / sqrt(mean(x[t, :]^2) + eps) in
// TO (fp16 for the tensor-core q_b_proj, fp32 for the CUDA-core one).
template <typename TO>
__global__ void __launch_bounds__(32 * kRowsPerNormBlock)
rmsnorm_f32_rows_kernel(const float* __restrict__ x, int splits, int64_t split_stride,
                        const __nv_bfloat16* __restrict__ w, TO* __restrict__ y, int64_t rows, int width, float eps) {
  const int64_t t = (int64_t)blockIdx.x * kRowsPerNormBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= rows) return;
  const float* xr = x + t * width;
  // x holds `splits` partial sums of the Linear, split_stride apart: added in split order
  auto xv = [&](int k) {
    float v = xr[k];
    for (int s = 1; s < splits; ++s) v += xr[(int64_t)s * split_stride + k];
    return v;
  };
  float ss = 0.f;
  for (int k = lane; k < width; k += 32) {
    const float v = xv(k);
    ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  const float r = 1.0f / sqrtf(ss / (float)width + eps);
  TO* yr = y + t * width;
  bool over = false;
  for (int k = lane; k < width; k += 32) {
    const float v = __bfloat162float(w[k]) * (xv(k) * r);
    if constexpr (sizeof(TO) == 2) {
      over |= !(fabsf(v) <= 65504.f);
      yr[k] = __float2half_rn(v);
    } else {
      yr[k] = v;
    }
  }
  if (over) raise_device_error(kDevErrRange);
}

// The joint down-projection's fp32 result x [n, R + P] of a bf16 run, one
// warp per token: latent[t] = bf16(x[t]) (compressed_kv, the prefill's latent
// input), and when `cache` is set the cache row
//   RMSNorm(x[t, :R]) || rope(x[t, R:], positions[t])
// into cache[cache_rows[t]], both computed from the fp32 values (the cache
// append of the GLM-5 "KV cache" section fused onto the Linear's result). x
// holds `splits` partial sums of the Linear, split_stride apart: the warp adds
// them in split order (16-byte loads, all of a lane's in flight) into its row
// in shared memory, and the rest reads the row from there. A destination row
// or position out of range skips the row's append and sets the device error
// word. R + P <= 768.
constexpr int kKvRowsPerBlock = 8;
constexpr int kKvMaxWidth = 768;
__global__ void __launch_bounds__(32 * kKvRowsPerBlock)
kv_latent_append_kernel(const float* __restrict__ x, int splits, int64_t split_stride,
                        __nv_bfloat16* __restrict__ latent, int64_t n, int R, int P,
                        const __nv_bfloat16* __restrict__ w_norm, const int32_t* __restrict__ positions,
                        const float* __restrict__ cos_t, const float* __restrict__ sin_t, int max_pos, int interleaved,
                        float eps, __nv_bfloat16* __restrict__ cache, int64_t cache_num_rows,
                        const int64_t* __restrict__ cache_rows) {
  __shared__ __align__(16) float s_row[kKvRowsPerBlock][kKvMaxWidth];
  const int wi = threadIdx.x >> 5;
  const int64_t t = (int64_t)blockIdx.x * kKvRowsPerBlock + wi;
  const int lane = threadIdx.x & 31;
  // the destination row and position are the caller's: read before the wait
  // for the Linear (launched as its programmatic dependent)
  const int64_t crow = (cache && t < n) ? cache_rows[t] : 0;
  const int64_t pos = (cache && t < n) ? positions[t] : 0;
  tc::pdl_wait();
  tc::pdl_allow_next();
  if (t >= n) return;
  const int W = R + P;
  const float* xr = x + t * W;
  float* row = s_row[wi];
  if (W % 4 == 0) {     // rows start on 16-byte boundaries
    const float4* x4 = reinterpret_cast<const float4*>(xr);
    const int64_t st4 = split_stride / 4;
#pragma unroll 4
    for (int c = lane; c < W / 4; c += 32) {
      float4 v = x4[c];
      for (int sp = 1; sp < splits; ++sp) {
        const float4 u = x4[sp * st4 + c];
        v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
      }
      reinterpret_cast<float4*>(row)[c] = v;
    }
  } else {
    for (int k = lane; k < W; k += 32) {
      float v = xr[k];
      for (int sp = 1; sp < splits; ++sp) v += xr[(int64_t)sp * split_stride + k];
      row[k] = v;
    }
  }
  __syncwarp();
  __nv_bfloat16* lr = latent + t * W;
  float ss = 0.f;
  for (int k = lane; k < W; k += 32) {
    const float v = row[k];
    lr[k] = __float2bfloat16_rn(v);
    if (k < R) ss = fmaf(v, v, ss);
  }
  if (!cache) return;
  ss = warp_sum(ss);
  if (crow < 0 || crow >= cache_num_rows || pos < 0 || pos >= max_pos) {
    if (lane == 0) raise_device_error(kDevErrBadInput);
    return;
  }
  const float r = 1.0f / sqrtf(ss / (float)R + eps);
  __nv_bfloat16* dst = cache + crow * W;
  for (int k = lane; k < R; k += 32) dst[k] = __float2bfloat16_rn(__bfloat162float(w_norm[k]) * (row[k] * r));
  const int half = P / 2;
  for (int i = lane; i < half; i += 32) {
    int a2, b2;
    rope_pair_slots(i, P, interleaved, a2, b2);
    float ox, oy;
    rope_turn(row[R + a2], row[R + b2], cos_t[pos * half + i], sin_t[pos * half + i], ox, oy);
    dst[R + a2] = __float2bfloat16_rn(ox);
    dst[R + b2] = __float2bfloat16_rn(oy);
  }
}

// out[t, j] = sum_k x[t, k] w[j, k], fp32 accumulation: 16 x 16 output tiles,
// K staged through shared memory 16 at a time. Every load is guarded. x, w
// and out may have different types (bf16 runs keep the results that feed an
// RMSNorm in fp32).
constexpr int kLinTile = 16;

template <typename T, typename TW = T, typename TO = T>
__global__ void __launch_bounds__(kLinTile * kLinTile)
simt_linear_kernel(const T* __restrict__ x, const TW* __restrict__ w, TO* __restrict__ out, int64_t n, int K,
                   int Nout) {
  __shared__ float sx[kLinTile][kLinTile + 1];
  __shared__ float sw[kLinTile][kLinTile + 1];
  const int tx = threadIdx.x % kLinTile, ty = threadIdx.x / kLinTile;
  const int64_t t = (int64_t)blockIdx.y * kLinTile + ty;   // output row
  const int j = blockIdx.x * kLinTile + tx;                  // output column
  const int64_t t_ld = (int64_t)blockIdx.y * kLinTile + ty;  // row of x this thread stages
  const int j_ld = blockIdx.x * kLinTile + ty;               // row of w this thread stages
  float acc = 0.f;
  for (int k0 = 0; k0 < K; k0 += kLinTile) {
    const int k = k0 + tx;
    sx[ty][tx] = (t_ld < n && k < K) ? to_f32(x[t_ld * K + k]) : 0.f;
    sw[ty][tx] = (j_ld < Nout && k < K) ? to_f32(w[(int64_t)j_ld * K + k]) : 0.f;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kLinTile; ++kk) acc = fmaf(sx[ty][kk], sw[tx][kk], acc);
    __syncthreads();
  }
  if (t < n && j < Nout) out[t * Nout + j] = from_f32<TO>(acc);
}

}  // namespace mla
