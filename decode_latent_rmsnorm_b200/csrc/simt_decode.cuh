// CUDA-core (FFMA) absorbed decode: exact fp32 arithmetic for MLA_FP32 runs
// and for head geometries the tensor-core decode does not take.
//
// Sources: GLM-5 "Normalized key-value latent" page, "KV cache" (the cache
// holds the normalized latent and the rotated shared key; heads come from
// kv_b_proj of every cached row) and the "Eager latent expansion" equation
// page, "Read the equation" (the absorbed path contracts the projection
// weights with the query and with the latent aggregate instead).
#pragma once
#include "common.cuh"

namespace mla {
namespace simt {

constexpr int kDecChunk = 2048;   // cache rows per split
constexpr int kDecTile = 16;      // cache rows staged per step
constexpr int kDecHeads = 16;     // heads per block

// q_lat[b, h, :] = W_UK_h^T q_nope[b, h] (fp32) and the rotated q_pe.
template <typename T>
__global__ void __launch_bounds__(256)
qprep_kernel(const T* __restrict__ q, const T* __restrict__ W, const int32_t* __restrict__ positions,
             const float* __restrict__ cos_t, const float* __restrict__ sin_t, int max_pos, int H,
             int R, int N, int P, int V, int interleaved, float* __restrict__ q_lat,
             float* __restrict__ q_rot) {
  __shared__ float qn[512];
  const int b = blockIdx.x, h = blockIdx.y;
  const int D = N + P;
  const T* qr = q + ((int64_t)b * H + h) * D;
  for (int j = threadIdx.x; j < N; j += blockDim.x) qn[j] = to_f32(qr[j]);
  __syncthreads();
  const T* Wk = W + (int64_t)h * (N + V) * R;        // rows of k_nope for head h
  for (int k = threadIdx.x; k < R; k += blockDim.x) {
    float a = 0.f;
    for (int j = 0; j < N; ++j) a = fmaf(to_f32(Wk[(int64_t)j * R + k]), qn[j], a);
    q_lat[((int64_t)b * H + h) * R + k] = a;
  }
  const int half = P / 2;
  const int64_t pos = checked_pos(positions[b], max_pos);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    int a, bb;
    rope_pair_slots(i, P, interleaved, a, bb);
    float ox, oy;
    rope_turn(to_f32(qr[N + a]), to_f32(qr[N + bb]), cos_t[pos * half + i], sin_t[pos * half + i],
              ox, oy);
    q_rot[((int64_t)b * H + h) * P + a] = ox;
    q_rot[((int64_t)b * H + h) * P + bb] = oy;
  }
}

// One block per (split, sequence, head group): running max / sum / latent
// aggregate over the split's rows. Partials are unnormalized and carry their
// own running max, merged by combine_kernel.
template <typename T>
__global__ void __launch_bounds__(256)
split_kernel(const float* __restrict__ q_lat, const float* __restrict__ q_rot,
             const T* __restrict__ cache, int64_t cache_num_rows, const int64_t* __restrict__ offsets,
             const int32_t* __restrict__ lens, int max_len, int H, int R, int P, float scale,
             int nsplit, float* __restrict__ o_part, float* __restrict__ m_part,
             float* __restrict__ l_part) {
  extern __shared__ float sm[];
  const int C = R + P;
  float* qs = sm;                          // [kDecHeads][C]
  float* cs = qs + kDecHeads * C;          // [kDecTile][C]
  float* ps = cs + kDecTile * C;           // [kDecHeads][kDecTile]
  const int split = blockIdx.x, b = blockIdx.y, h0 = blockIdx.z * kDecHeads;
  const int tid = threadIdx.x;
  const int64_t off = offsets[b];
  int L = lens[b];
  if (L < 1 || L > max_len || off < 0 || off + L > cache_num_rows) {   // bad sequence: skipped
    if (split == 0 && blockIdx.z == 0 && tid == 0) raise_device_error(kDevErrBadInput);
    L = 0;
  }
  const int r0 = split * kDecChunk, r1 = min(L, r0 + kDecChunk);
  const int hh = tid >> 4, sub = tid & 15;
  const int h = h0 + hh;
  const bool hv = h < H;

  for (int e = tid; e < kDecHeads * C; e += 256) {
    const int x = e / C, d = e % C, hx = h0 + x;
    float v = 0.f;
    if (hx < H) v = d < R ? q_lat[((int64_t)b * H + hx) * R + d] : q_rot[((int64_t)b * H + hx) * P + d - R];
    qs[e] = v;
  }
  float m = -INFINITY, l = 0.f;
  float acc[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) acc[c] = 0.f;
  const int nk = R / 16;
  const T* base = cache + (L > 0 ? off : 0) * C;

  for (int t0 = r0; t0 < r1; t0 += kDecTile) {
    __syncthreads();
    for (int e = tid; e < kDecTile * C; e += 256) {
      const int r = e / C, d = e % C;
      cs[e] = (t0 + r < r1) ? to_f32(base[(int64_t)(t0 + r) * C + d]) : 0.f;
    }
    __syncthreads();
    float s = -INFINITY;
    if (t0 + sub < r1) {
      float a = 0.f;
      for (int d = 0; d < C; ++d) a = fmaf(qs[hh * C + d], cs[sub * C + d], a);
      s = a * scale;
    }
    float tmax = s;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float m_new = fmaxf(m, tmax);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
    const float p = (s == -INFINITY) ? 0.f : expf(s - m_new);
    float psum = p;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    ps[hh * kDecTile + sub] = p;
    __syncthreads();
    m = m_new;
    l = l * alpha + psum;
    for (int c = 0; c < nk; ++c) {
      const int k = sub + 16 * c;
      float a = acc[c] * alpha;
#pragma unroll
      for (int r = 0; r < kDecTile; ++r) a = fmaf(ps[hh * kDecTile + r], cs[r * C + k], a);
      acc[c] = a;
    }
  }
  if (hv) {
    const int64_t slot = ((int64_t)b * nsplit + split) * H + h;
    for (int c = 0; c < nk; ++c) o_part[slot * R + sub + 16 * c] = acc[c];
    if (sub == 0) { m_part[slot] = m; l_part[slot] = l; }
  }
}

inline size_t split_smem_bytes(int R, int P) {
  return sizeof(float) * ((size_t)(kDecHeads + kDecTile) * (R + P) + kDecHeads * kDecTile);
}

// Merge the splits of (b, h) by their log-sum-exp, then out = W_UV_h o_lat.
template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ o_part, const float* __restrict__ m_part,
               const float* __restrict__ l_part, const T* __restrict__ W, int H, int R, int N, int V,
               int nsplit, T* __restrict__ out) {
  __shared__ float ol[1024];
  __shared__ float wsplit[256];
  const int b = blockIdx.x, h = blockIdx.y;
  const int64_t slot0 = (int64_t)b * nsplit * H + h;   // slot of split s: slot0 + s*H
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, m_part[slot0 + (int64_t)s * H]);
  float Lsum = 0.f;
  for (int s = threadIdx.x; s < nsplit; s += blockDim.x) {
    const float ms = m_part[slot0 + (int64_t)s * H];
    wsplit[s] = (ms == -INFINITY) ? 0.f : expf(ms - M);
  }
  __syncthreads();
  for (int s = 0; s < nsplit; ++s) Lsum += wsplit[s] * l_part[slot0 + (int64_t)s * H];
  if (!(Lsum > 0.f)) {   // a skipped sequence: no row to attend (flagged by split_kernel)
    for (int c = threadIdx.x; c < V; c += blockDim.x) out[((int64_t)b * H + h) * V + c] = from_f32<T>(0.f);
    return;
  }
  for (int k = threadIdx.x; k < R; k += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < nsplit; ++s) a = fmaf(wsplit[s], o_part[(slot0 + (int64_t)s * H) * R + k], a);
    ol[k] = a / Lsum;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* Wv = W + ((int64_t)h * (N + V) + N) * R;   // value rows of head h
  for (int c = warp; c < V; c += 8) {
    float a = 0.f;
    for (int k = lane; k < R; k += 32) a = fmaf(to_f32(Wv[(int64_t)c * R + k]), ol[k], a);
    a = warp_sum(a);
    if (lane == 0) out[((int64_t)b * H + h) * V + c] = from_f32<T>(a);
  }
}

}  // namespace simt
}  // namespace mla
