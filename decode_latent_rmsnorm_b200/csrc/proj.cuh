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
#include "common.cuh"

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

// out[t, j] = sum_k x[t, k] w[j, k], fp32 accumulation: 16 x 16 output tiles,
// K staged through shared memory 16 at a time. Every load is guarded.
constexpr int kLinTile = 16;

template <typename T>
__global__ void __launch_bounds__(kLinTile * kLinTile)
simt_linear_kernel(const T* __restrict__ x, const T* __restrict__ w, T* __restrict__ out, int64_t n, int K,
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
  if (t < n && j < Nout) out[t * Nout + j] = from_f32<T>(acc);
}

}  // namespace mla
