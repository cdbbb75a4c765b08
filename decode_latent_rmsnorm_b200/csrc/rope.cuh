// Rotary coefficient tables (Kimi-K2 "RoPE coefficients" page, "Generate
// RoPE coefficients": YaRN correction range, linear ramp between base and
// interpolated frequencies, cos/sin tables scaled by the ratio of the two
// YaRN corrections).
#pragma once
#include "common.cuh"

namespace mla {

struct RopeTableParams {
  int pairs;             // rope_dim / 2
  int rope_dim;
  int yarn;
  double base, factor;
  double ramp_lo, ramp_hi;   // correction range (hi already nudged if equal)
  double table_mscale;
};

// One thread per (position, pair). The frequency and the angle are formed in
// fp64 so the only rounding in the table is its final fp32 store.
__global__ void rope_tables_kernel(RopeTableParams p, int max_pos, float* __restrict__ cos_t,
                                   float* __restrict__ sin_t) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = (int64_t)max_pos * p.pairs;
  if (idx >= n) return;
  const int pos = (int)(idx / p.pairs);
  const int i = (int)(idx % p.pairs);
  const double e = (2.0 * i) / (double)p.rope_dim;
  const double base_freq = 1.0 / pow(p.base, e);
  double inv_freq = base_freq;
  if (p.yarn) {
    // Pairs below the range keep the base frequency, pairs above it are
    // divided by the factor, pairs inside are blended linearly.
    double ramp = ((double)i - p.ramp_lo) / (p.ramp_hi - p.ramp_lo);
    ramp = ramp < 0.0 ? 0.0 : (ramp > 1.0 ? 1.0 : ramp);
    const double interp = base_freq / p.factor;
    inv_freq = interp * ramp + base_freq * (1.0 - ramp);
  }
  const double ang = (double)pos * inv_freq;
  cos_t[idx] = (float)(cos(ang) * p.table_mscale);
  sin_t[idx] = (float)(sin(ang) * p.table_mscale);
}

}  // namespace mla
