// C-ABI of the MLA hot path (declared in include/mla.h). Host-side argument
// checks, workspace carving and kernel launches; every step of the path runs
// in the kernels included below.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>

#include "mla.h"
#include "common.cuh"
#include "rope.cuh"
#include "simt_prefill.cuh"
#include "simt_decode.cuh"
#include "tc_gemm.cuh"
#include "tc_attention.cuh"
#include "tc_attention_pair.cuh"
#include "tc_decode.cuh"
#include "chunk.cuh"
#include "tc_chunk.cuh"
#include "tc_linear.cuh"
#include "proj.cuh"
#include "selftest.cuh"

#include <cudaTypedefs.h>

// Scratch of mla_prefill_noalloc: the workspace for callers that cannot
// allocate. It lives on every device that loads this library.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];

namespace {

thread_local char g_err[1024] = "no error";
// Which kernels the last prefill / decode call of this thread ran, and why
// (mla_last_dispatch).
thread_local const char* g_dispatch = "none";
void set_dispatch(const char* what) { g_dispatch = what; }

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

// A failed launch also leaves its error in the runtime's last-error slot;
// reading the slot here clears it, so that the error is reported once, by the
// call that made it, and not again by the next call's launch check.
int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MLA_OK;
  (void)cudaGetLastError();
  return fail(MLA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- TMA tensor maps (driver entry point fetched through the runtime) --------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode() {
  if (g_encode) return MLA_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
    return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return MLA_OK;
}

// 16-bit tensor map with the 128-byte swizzle; dims/strides innermost first
// (strides in bytes, for dims 1..rank-1).
int make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
             const uint32_t* box, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  int rc = get_encode();
  if (rc) return rc;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) { d[i] = dims[i]; b[i] = box[i]; es[i] = 1; }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides[i];
  CUresult r = g_encode(m, dtype, rank, const_cast<void*>(base), d, st, b, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

// ---- launch accounting and optional per-kernel events ---------------------
std::atomic<uint64_t> g_launches{0};
thread_local cudaEvent_t const* g_events = nullptr;
thread_local int g_event_pairs = 0;
thread_local int g_event_next = 0;
constexpr int kMaxNamed = 256;
thread_local const char* g_event_names[kMaxNamed];

// Bracket one kernel launch: prof_begin before, prof_end after.
void prof_begin(cudaStream_t st, const char* name) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_events && g_event_next < g_event_pairs) {
    if (g_event_next < kMaxNamed) g_event_names[g_event_next] = name;
    cudaEventRecord(g_events[2 * g_event_next], st);
  }
}
void prof_end(cudaStream_t st) {
  if (g_events && g_event_next < g_event_pairs) {
    cudaEventRecord(g_events[2 * g_event_next + 1], st);
    ++g_event_next;
  }
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel of the stream is finishing; it waits in device code
// (pdl_wait) before it reads that kernel's results. Used for the second and
// later kernels of one call.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- YaRN scalars (Kimi-K2 "RoPE coefficients" page, rope excerpt) -------
double correction_dim(double rotations, int dim, double base, double max_pos) {
  return (dim * log(max_pos / (rotations * 2.0 * M_PI))) / (2.0 * log(base));
}
double yarn_mscale(double scale, double m) {
  return scale <= 1.0 ? 1.0 : 0.1 * m * log(scale) + 1.0;
}

int check_rope(const mla_rope_cfg* r) {
  if (!r) return fail(MLA_ERR_INVALID_ARG, "rope config is NULL");
  if (r->rope_dim < 2 || r->rope_dim > 256 || (r->rope_dim & 1))
    return fail(MLA_ERR_INVALID_ARG, "rope_dim must be even and in [2, 256], got %d", r->rope_dim);
  if (!(r->base > 1.0)) return fail(MLA_ERR_INVALID_ARG, "rope base must be > 1");
  if (r->yarn != 0 && r->yarn != 1) return fail(MLA_ERR_INVALID_ARG, "yarn must be 0 or 1");
  if (r->reserved != 0) return fail(MLA_ERR_INVALID_ARG, "reserved field must be 0");
  if (r->yarn) {
    if (!(r->factor > 0.0)) return fail(MLA_ERR_INVALID_ARG, "YaRN factor must be > 0");
    if (r->original_max_pos < 1) return fail(MLA_ERR_INVALID_ARG, "original_max_pos must be >= 1");
    if (!(r->beta_fast > 0.0) || !(r->beta_slow > 0.0))
      return fail(MLA_ERR_INVALID_ARG, "beta_fast and beta_slow must be > 0");
  }
  return MLA_OK;
}

int check_dims(const mla_dims* d) {
  if (!d) return fail(MLA_ERR_INVALID_ARG, "dims is NULL");
  if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32)
    return fail(MLA_ERR_INVALID_ARG, "dtype must be MLA_BF16 (0) or MLA_FP32 (1), got %d", d->dtype);
  if (d->num_heads < 1 || d->kv_lora_rank < 1 || d->qk_nope < 0 || d->qk_rope < 2 || d->v_head < 1)
    return fail(MLA_ERR_INVALID_ARG, "non-positive head geometry");
  if (d->qk_rope & 1) return fail(MLA_ERR_INVALID_ARG, "qk_rope must be even");
  if (d->rope_interleaved != 0 && d->rope_interleaved != 1)
    return fail(MLA_ERR_INVALID_ARG, "rope_interleaved must be 0 or 1");
  if (!(d->eps >= 0.0f)) return fail(MLA_ERR_INVALID_ARG, "eps must be >= 0");
  if (!(d->softmax_scale > 0.0f) || !isfinite(d->softmax_scale))
    return fail(MLA_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (d->kv_lora_rank % 16 || d->kv_lora_rank > 512)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "kv_lora_rank must be a multiple of 16 and <= 512");
  if (d->v_head % 8 || d->v_head > 256)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "v_head must be a multiple of 8 and <= 256");
  if (d->qk_nope + d->qk_rope > 512 || d->qk_rope > 256)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "qk head dim must be <= 512 and qk_rope <= 256");
  return MLA_OK;
}

size_t elem_size(const mla_dims* d) { return d->dtype == MLA_FP32 ? 4 : 2; }

// Shapes the tensor-core prefill takes (bf16; otherwise the SIMT kernels run).
bool prefill_tc_shape(const mla_dims* d) {
  return d->dtype == MLA_BF16 && d->kv_lora_rank % 64 == 0 && d->kv_lora_rank <= 512 && d->qk_nope % 64 == 0 &&
         d->qk_nope >= 64 && d->qk_rope == 64 && d->v_head % 64 == 0 && d->v_head <= 256 &&
         d->qk_nope + d->qk_rope <= 256;
}

// SIMT prefill workspace: k_nope [H, Ttot, N], values [H, Ttot, V], k_rot [Ttot, P].
// Tensor-core workspace: tile schedule, then the padded k_nope [H, Tpad, N],
// transposed values [H, V, Tpad] and k_rot [Tpad, P], with Tpad = 128 * cap
// and cap = ceil(Ttot / 128) + num_seqs bounding the number of 128-row tiles.
struct PrefillWs {
  int64_t cap, Tpad;
  int gemm_tiles_per_cta, gemm_gy;
  size_t seq_tile0, tile_seq, tile_q0, order, pair_order, item_counter, w16, c16, q_rope;
  size_t k_nope, vals, k_rot, total;
};
PrefillWs prefill_ws_layout(const mla_dims* d, int64_t T, int nseq, bool tc) {
  PrefillWs w = {};
  const size_t es = elem_size(d);
  size_t off = 0;
  if (tc) {
    w.cap = (T + 127) / 128 + nseq;
    w.Tpad = w.cap * 128;
    // GEMM grid: (cap, gy) CTAs, each with tiles_per_cta output tiles of 256 columns
    const int NOUT = d->num_heads * (d->qk_nope + d->v_head);
    const int n_total = (NOUT + mla::tc::kGemmBN - 1) / mla::tc::kGemmBN;
    int splits = (int)(148 / (w.cap > 0 ? w.cap : 1));
    if (splits < 1) splits = 1;
    if (splits > n_total) splits = n_total;
    w.gemm_tiles_per_cta = (n_total + splits - 1) / splits;
    w.gemm_gy = (n_total + w.gemm_tiles_per_cta - 1) / w.gemm_tiles_per_cta;
    w.seq_tile0 = off; off = align_up(off + 4 * (size_t)(nseq + 1), 256);
    w.tile_seq = off;  off = align_up(off + 4 * (size_t)w.cap, 256);
    w.tile_q0 = off;   off = align_up(off + 4 * (size_t)w.cap, 256);
    w.order = off;     off = align_up(off + 4 * (size_t)w.cap, 256);
    w.pair_order = off; off = align_up(off + 4 * (size_t)w.cap, 256);
    w.item_counter = off; off = align_up(off + 4, 256);
    w.w16 = off;       off = align_up(off + 2 * (size_t)NOUT * d->kv_lora_rank, 256);
    w.c16 = off;       off = align_up(off + 2 * (size_t)T * d->kv_lora_rank, 256);   // normalized latent, fp16
    w.q_rope = off;    off = align_up(off + 2 * (size_t)T * d->num_heads * d->qk_rope, 256);   // rotated q, fp16
  } else {
    w.Tpad = T;
  }
  const size_t Tp = (size_t)w.Tpad;
  w.k_nope = off; off = align_up(off + es * (size_t)d->num_heads * Tp * d->qk_nope, 256);
  w.vals = off;   off = align_up(off + es * (size_t)d->num_heads * Tp * d->v_head, 256);
  w.k_rot = off;  off = align_up(off + es * Tp * d->qk_rope, 256);
  w.total = off;
  return w;
}
size_t prefill_ws_bytes(const mla_dims* d, int64_t T, int nseq) {
  size_t a = prefill_ws_layout(d, T, nseq, false).total;
  if (prefill_tc_shape(d)) {
    const size_t b = prefill_ws_layout(d, T, nseq, true).total;
    if (b > a) a = b;
  }
  return a;
}

// Shapes the tensor-core decode takes (bf16, 64 heads, 512 + 64 latent row).
// Up to 64 heads: fewer heads (a head-sharded decode) are padded to 64 with
// zero queries, whose outputs are never un-absorbed; the kernel streams the
// same cache bytes either way.
bool decode_tc_shape(const mla_dims* d) {
  return d->dtype == MLA_BF16 && d->num_heads >= 1 && d->num_heads <= mla::tc::kDecHeads && d->kv_lora_rank == 512 &&
         d->qk_rope == 64 && d->qk_nope % 64 == 0 && d->qk_nope >= 64;
}

int g_num_sms[64] = {};
int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!g_num_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

// SIMT decode workspace: q_lat [B, H, R], q_rot [B, H, P], per-split partials.
// Tensor-core decode workspace: prefix [B + 1] and meta [2] (int64), q [B, H,
// R + P] bf16, partials of B + G slots, o_lat [B, H, R] fp32.
struct DecodeWs {
  int nsplit;
  size_t q_lat, q_rot, o_part, m_part, l_part, total;
  size_t prefix, meta, qf, o_lat;
  int G;
};
DecodeWs decode_ws_layout(const mla_dims* d, int B, int max_len, bool tc) {
  DecodeWs w = {};
  const size_t H = d->num_heads, R = d->kv_lora_rank, P = d->qk_rope;
  size_t off = 0;
  if (tc) {
    const size_t Hp = mla::tc::kDecHeads;   // heads padded to the kernel's 64
    w.G = num_sms();
    const size_t slots = (size_t)B + w.G;
    w.prefix = off; off = align_up(off + 8 * (size_t)(B + 1), 256);
    w.meta = off;   off = align_up(off + 16, 256);
    w.qf = off;     off = align_up(off + 2 * (size_t)B * Hp * (R + P), 256);
    w.o_part = off; off = align_up(off + 4 * slots * Hp * R, 256);
    w.m_part = off; off = align_up(off + 4 * slots * Hp, 256);
    w.l_part = off; off = align_up(off + 4 * slots * Hp, 256);
    w.o_lat = off;  off = align_up(off + 2 * (size_t)B * Hp * R, 256);
    w.total = off;
    return w;
  }
  w.nsplit = (max_len + mla::simt::kDecChunk - 1) / mla::simt::kDecChunk;
  if (w.nsplit < 1) w.nsplit = 1;
  const size_t S = w.nsplit;
  w.q_lat = off;  off = align_up(off + 4 * (size_t)B * H * R, 256);
  w.q_rot = off;  off = align_up(off + 4 * (size_t)B * H * P, 256);
  w.o_part = off; off = align_up(off + 4 * (size_t)B * S * H * R, 256);
  w.m_part = off; off = align_up(off + 4 * (size_t)B * S * H, 256);
  w.l_part = off; off = align_up(off + 4 * (size_t)B * S * H, 256);
  w.total = off;
  return w;
}
size_t decode_ws_bytes(const mla_dims* d, int B, int max_len) {
  size_t a = decode_ws_layout(d, B, max_len, false).total;
  if (decode_tc_shape(d)) {
    const size_t b = decode_ws_layout(d, B, max_len, true).total;
    if (b > a) a = b;
  }
  return a;
}

template <typename T>
int launch_prefill(const mla_dims* d, const void* latent, const void* q, const void* w_kvb,
                   const void* w_norm, const int32_t* positions, const int32_t* cu_seqlens,
                   int num_seqs, int max_seqlen, int64_t T_tot, const float* cos_t,
                   const float* sin_t, int max_pos, void* out, void* workspace, cudaStream_t st) {
  using namespace mla::simt;
  const int H = d->num_heads, R = d->kv_lora_rank, N = d->qk_nope, P = d->qk_rope, V = d->v_head;
  const PrefillWs L = prefill_ws_layout(d, T_tot, num_seqs, false);
  char* ws = static_cast<char*>(workspace);
  T* k_nope = reinterpret_cast<T*>(ws + L.k_nope);
  T* vals = reinterpret_cast<T*>(ws + L.vals);
  T* k_rot = reinterpret_cast<T*>(ws + L.k_rot);
  const int NOUT = H * (N + V);
  dim3 g1((unsigned)((T_tot + kGemmBM - 1) / kGemmBM), (unsigned)((NOUT + kGemmBN - 1) / kGemmBN));
  prof_begin(st, "simt_norm_kv_b_proj");
  norm_proj_kernel<T><<<g1, 256, 0, st>>>(static_cast<const T*>(latent), static_cast<const T*>(w_kvb),
                                          static_cast<const T*>(w_norm), T_tot, R, P, H, N, V, d->eps,
                                          k_nope, vals);
  prof_end(st);
  const int64_t npairs = T_tot * (P / 2);
  prof_begin(st, "simt_rope_key");
  rope_key_kernel<T><<<(unsigned)((npairs + 255) / 256), 256, 0, st>>>(
      static_cast<const T*>(latent), positions, cos_t, sin_t, max_pos, T_tot, R, P, d->rope_interleaved,
      k_rot);
  prof_end(st);
  const size_t smem = attention_smem_bytes(N + P, V);
  cudaError_t e = cudaFuncSetAttribute(attention_kernel<T, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return cuda_status(e, "attention smem attribute");
  dim3 g2((unsigned)((max_seqlen + kAttBQ - 1) / kAttBQ), (unsigned)num_seqs, (unsigned)H);
  prof_begin(st, "simt_attention");
  attention_kernel<T, false><<<g2, 256, smem, st>>>(static_cast<const T*>(q), k_nope, k_rot, vals, positions,
                                                    cu_seqlens, cos_t, sin_t, max_pos, max_seqlen, T_tot, H, N, P,
                                                    V, d->rope_interleaved, d->softmax_scale, static_cast<T*>(out),
                                                    nullptr, T_tot);
  prof_end(st);
  return cuda_status(cudaGetLastError(), "prefill launch");
}

template <int kN, int kV>
int launch_attention_tc_t(unsigned grid, const CUtensorMap& mq, const CUtensorMap& mqr, const CUtensorMap& mkn,
                          const CUtensorMap& mkr, const CUtensorMap& mvt, const mla::tc::AttParams& ap,
                          cudaStream_t st) {
  // deepest K/V pipeline that fits next to Q and P in 227 KB of shared memory
  constexpr size_t kBase = mla::tc::AttCfg<kN, kV, 1>::kSmem - mla::tc::AttCfg<kN, kV, 1>::kStageBytes;
  constexpr size_t kStage = mla::tc::AttCfg<kN, kV, 1>::kStageBytes;
  constexpr int kFit = (int)((232448 - 1024 - kBase) / kStage);
  constexpr int kStages = kFit >= 3 ? 3 : 2;
  static_assert(kFit >= 2, "attention tile does not fit in shared memory");
  using C = mla::tc::AttCfg<kN, kV, kStages>;
  auto kern = mla::tc::attention_kernel<kN, kV, kStages>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (e != cudaSuccess) return cuda_status(e, "attention smem attribute");
  prof_begin(st, "tc_attention");
  e = launch_dependent(kern, dim3(grid), dim3(mla::tc::kAttThreads), C::kSmem, st, mq, mqr, mkn, mkr, mvt, ap);
  prof_end(st);
  return cuda_status(e, "attention launch");
}

int launch_attention_tc(int N, int V, unsigned grid, const CUtensorMap& mq, const CUtensorMap& mqr,
                        const CUtensorMap& mkn, const CUtensorMap& mkr, const CUtensorMap& mvt,
                        const mla::tc::AttParams& ap, cudaStream_t st) {
#define MLA_ATT_CASE(n, v) \
  if (N == n && V == v) return launch_attention_tc_t<n, v>(grid, mq, mqr, mkn, mkr, mvt, ap, st);
  MLA_ATT_CASE(64, 64) MLA_ATT_CASE(64, 128) MLA_ATT_CASE(64, 192) MLA_ATT_CASE(64, 256)
  MLA_ATT_CASE(128, 64) MLA_ATT_CASE(128, 128) MLA_ATT_CASE(128, 192) MLA_ATT_CASE(128, 256)
  MLA_ATT_CASE(192, 64) MLA_ATT_CASE(192, 128) MLA_ATT_CASE(192, 192) MLA_ATT_CASE(192, 256)
#undef MLA_ATT_CASE
  return fail(MLA_ERR_UNSUPPORTED_SHAPE, "no tensor-core attention for qk_nope=%d v_head=%d", N, V);
}

// Head geometries of the two-tile attention kernel (two fp32 O accumulators
// of V columns next to two 128-column S buffers in 512 TMEM columns).
bool attention_pair_shape(int N, int V) { return (N == 64 || N == 128) && (V == 64 || V == 128); }

template <int kN, int kV>
int launch_attention_pair_t(unsigned grid, const CUtensorMap& mq, const CUtensorMap& mqr, const CUtensorMap& mkn,
                            const CUtensorMap& mkr, const CUtensorMap& mvt, const mla::tc::AttParams& ap,
                            cudaStream_t st) {
  using C = mla::tc::PairCfg<kN, kV>;
  auto kern = mla::tc::attention_pair_kernel<kN, kV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (e != cudaSuccess) return cuda_status(e, "attention smem attribute");
  prof_begin(st, "tc_attention");
  e = launch_dependent(kern, dim3(grid), dim3(mla::tc::kPrThreads), C::kSmem, st, mq, mqr, mkn, mkr, mvt, ap);
  prof_end(st);
  return cuda_status(e, "attention launch");
}

int launch_attention_pair(int N, int V, unsigned grid, const CUtensorMap& mq, const CUtensorMap& mqr,
                          const CUtensorMap& mkn, const CUtensorMap& mkr, const CUtensorMap& mvt,
                          const mla::tc::AttParams& ap, cudaStream_t st) {
#define MLA_PAIR_CASE(n, v) \
  if (N == n && V == v) return launch_attention_pair_t<n, v>(grid, mq, mqr, mkn, mkr, mvt, ap, st);
  MLA_PAIR_CASE(64, 64) MLA_PAIR_CASE(64, 128) MLA_PAIR_CASE(128, 64) MLA_PAIR_CASE(128, 128)
#undef MLA_PAIR_CASE
  return fail(MLA_ERR_UNSUPPORTED_SHAPE, "no two-tile attention for qk_nope=%d v_head=%d", N, V);
}

// Tensor-core prefill: tile schedule -> fused RMSNorm + kv_b_proj (tcgen05)
// -> causal attention over the padded layout.
// w_f16: the fp16 copy of w_kvb made by mla_prepare_kv_b_proj, or NULL to make
// it here (in the workspace) on every call.
int launch_prefill_tc(const mla_dims* d, const void* latent, const void* q, const void* w_kvb, const void* w_f16,
                      const void* w_norm, const int32_t* positions, const int32_t* cu_seqlens, int num_seqs,
                      int max_seqlen, int64_t T_tot, const float* cos_t, const float* sin_t, int max_pos,
                      void* out, void* workspace, cudaStream_t st) {
  using bf16 = __nv_bfloat16;
  const int H = d->num_heads, R = d->kv_lora_rank, N = d->qk_nope, P = d->qk_rope, V = d->v_head;
  const PrefillWs L = prefill_ws_layout(d, T_tot, num_seqs, true);
  char* ws = static_cast<char*>(workspace);
  int32_t* seq_tile0 = reinterpret_cast<int32_t*>(ws + L.seq_tile0);
  int32_t* tile_seq = reinterpret_cast<int32_t*>(ws + L.tile_seq);
  int32_t* tile_q0 = reinterpret_cast<int32_t*>(ws + L.tile_q0);
  int32_t* order = reinterpret_cast<int32_t*>(ws + L.order);
  int32_t* pair_order = reinterpret_cast<int32_t*>(ws + L.pair_order);
  int32_t* item_counter = reinterpret_cast<int32_t*>(ws + L.item_counter);
  __half* k_nope = reinterpret_cast<__half*>(ws + L.k_nope);
  __half* vt = reinterpret_cast<__half*>(ws + L.vals);
  __half* k_rot = reinterpret_cast<__half*>(ws + L.k_rot);
  __half* q_rope = reinterpret_cast<__half*>(ws + L.q_rope);
  const int cap = (int)L.cap;
  const int NOUT = H * (N + V);
  // both attention kernels take k_nope in bf16 and the queries' rotated part
  // from the preparation kernel
  const bool pair = attention_pair_shape(N, V) && d->softmax_scale > 0.f;

  CUtensorMap map_lat, map_w;
  {
    const uint64_t dims[2] = {(uint64_t)(R + P), (uint64_t)T_tot};
    const uint64_t strides[1] = {(uint64_t)(R + P) * 2};
    const uint32_t box[2] = {64, 128};
    int rc = make_map(&map_lat, latent, 2, dims, strides, box);
    if (rc) return rc;
  }
  // heads with V = 128 and qk_nope 64 or 128 take the GEMM that writes the
  // value half transposed straight from TMEM (one head's weight rows per stage)
  const bool vt_gemm = (N == 64 || N == 128) && V == 128;
  {
    const uint64_t dims[2] = {(uint64_t)R, (uint64_t)NOUT};
    const uint64_t strides[1] = {(uint64_t)R * 2};
    const uint32_t box[2] = {64, vt_gemm ? (uint32_t)(N + V) : 256u};
    int rc = make_map(&map_w, w_f16 ? w_f16 : (const void*)(ws + L.w16), 2, dims, strides, box,
                      CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }

  __half* w16 = reinterpret_cast<__half*>(ws + L.w16);
  const int gy = L.gemm_gy;

  __half* c16 = reinterpret_cast<__half*>(ws + L.c16);
  const int64_t n8 = (int64_t)NOUT * R / 8;
  const int64_t per_block = (int64_t)mla::tc::kPrepThreads * mla::tc::kPrepUnroll;
  const int w_blocks = w_f16 ? 0 : (int)((n8 + per_block - 1) / per_block);
  // the transposed-value GEMM reads c_hat prepared here: one warp per token row
  const int norm_blocks = vt_gemm ? (int)((T_tot + mla::tc::kPrepThreads / 32 - 1) / (mla::tc::kPrepThreads / 32)) : 0;
  mla::tc::QRopeParams qrp{};
  qrp.q = static_cast<const bf16*>(q);
  qrp.positions = positions;
  qrp.cos_t = cos_t;
  qrp.sin_t = sin_t;
  qrp.qr = q_rope;
  qrp.rows = T_tot * H;
  qrp.H = H; qrp.D = N + P; qrp.N = N; qrp.max_pos = max_pos; qrp.interleaved = d->rope_interleaved;
  const int qr_blocks = (int)mla::tc::q_rope_blocks(qrp.rows, H, mla::tc::kPrepThreads);
  prof_begin(st, "tc_prep");
  mla::tc::prefill_prep_kernel<<<(unsigned)(1 + w_blocks + norm_blocks + qr_blocks), mla::tc::kPrepThreads, 0,
                                 st>>>(
      cu_seqlens, num_seqs, T_tot, max_seqlen, cap, seq_tile0, tile_seq, tile_q0, order, pair_order,
      item_counter, static_cast<const bf16*>(w_kvb), w16, n8, w_blocks, static_cast<const bf16*>(latent),
      static_cast<const bf16*>(w_norm), R, d->eps, c16, norm_blocks, qrp);
  prof_end(st);
  CUtensorMap map_c16;   // the transposed-value GEMM's A operand: c_hat fp16 [Ttot, R]
  {
    const uint64_t dims[2] = {(uint64_t)R, (uint64_t)T_tot};
    const uint64_t strides[1] = {(uint64_t)R * 2};
    const uint32_t box[2] = {64, 128};
    int rc = make_map(&map_c16, c16, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }

  mla::tc::GemmParams gp{};
  gp.latent = static_cast<const bf16*>(latent);
  gp.w_norm = static_cast<const bf16*>(w_norm);
  gp.positions = positions;
  gp.cu = cu_seqlens;
  gp.tile_seq = tile_seq;
  gp.tile_q0 = tile_q0;
  gp.cos_t = cos_t;
  gp.sin_t = sin_t;
  gp.k_nope = k_nope;
  gp.vt = vt;
  gp.k_rot = k_rot;
  gp.Ttot = T_tot;
  gp.Tpad = (int)L.Tpad;
  gp.R = R; gp.P = P; gp.H = H; gp.N = N; gp.V = V; gp.NOUT = NOUT;
  gp.max_pos = max_pos;
  gp.interleaved = d->rope_interleaved;
  gp.eps = d->eps;
  gp.tiles_per_cta = L.gemm_tiles_per_cta;
  gp.knope_bf16 = 1;
  cudaError_t e;
  if (vt_gemm) {
    // grid: (tiles, head groups); about one CTA per SM over the real tiles
    const int real_tiles = (int)((T_tot + 127) / 128) + (num_seqs > 1 ? num_seqs - 1 : 0);
    int groups = num_sms() / (real_tiles > 0 ? real_tiles : 1);
    if (groups < 1) groups = 1;
    if (groups > H) groups = H;
    gp.tiles_per_cta = (H + groups - 1) / groups;
    const int gy2 = (H + gp.tiles_per_cta - 1) / gp.tiles_per_cta;
    auto kern = N == 64 ? mla::tc::norm_kvb_gemm_vt_kernel<64> : mla::tc::norm_kvb_gemm_vt_kernel<128>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mla::tc::kG2SmemBytes);
    if (e != cudaSuccess) return cuda_status(e, "gemm smem attribute");
    prof_begin(st, "tc_norm_kv_b_proj");
    e = launch_dependent(kern, dim3(cap, gy2), dim3(mla::tc::kG2Threads), mla::tc::kG2SmemBytes, st, map_c16, map_w,
                         gp);
    prof_end(st);
    if (e != cudaSuccess) return cuda_status(e, "gemm launch");
  } else {
    e = cudaFuncSetAttribute(mla::tc::norm_kvb_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)mla::tc::kGemmSmemBytes);
    if (e != cudaSuccess) return cuda_status(e, "gemm smem attribute");
    prof_begin(st, "tc_norm_kv_b_proj");
    e = launch_dependent(mla::tc::norm_kvb_gemm_kernel, dim3(cap, gy), dim3(mla::tc::kGemmThreads),
                         mla::tc::kGemmSmemBytes, st, map_lat, map_w, gp);
    prof_end(st);
    if (e != cudaSuccess) return cuda_status(e, "gemm launch");
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "gemm launch");

  // attention tensor maps over the padded workspace, q [Ttot, H, D] and the
  // rotated q [Ttot, H, P]; the two-tile kernel reads 128 keys per step, the
  // one-tile kernel 64
  const uint32_t kv_box = pair ? (uint32_t)mla::tc::kPrBKV : (uint32_t)mla::tc::kAttBKV;
  const int D = N + P;
  CUtensorMap map_q, map_qr, map_kn, map_kr, map_vt;
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)H, (uint64_t)T_tot};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)H * D * 2};
    const uint32_t box[3] = {64, 1, 128};
    int rc = make_map(&map_q, q, 3, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {(uint64_t)P, (uint64_t)H, (uint64_t)T_tot};
    const uint64_t strides[2] = {(uint64_t)P * 2, (uint64_t)H * P * 2};
    const uint32_t box[3] = {64, 1, 128};
    int rc = make_map(&map_qr, q_rope, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)H * L.Tpad};
    const uint64_t strides[1] = {(uint64_t)N * 2};
    const uint32_t box[2] = {64, kv_box};
    int rc = make_map(&map_kn, k_nope, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)P, (uint64_t)L.Tpad};
    const uint64_t strides[1] = {(uint64_t)P * 2};
    const uint32_t box[2] = {64, kv_box};
    int rc = make_map(&map_kr, k_rot, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)L.Tpad, (uint64_t)H * V};
    const uint64_t strides[1] = {(uint64_t)L.Tpad * 2};
    const uint32_t box[2] = {64, (uint32_t)V};
    int rc = make_map(&map_vt, vt, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  mla::tc::AttParams ap;
  ap.cu = cu_seqlens;
  ap.positions = positions;
  ap.seq_tile0 = seq_tile0;
  ap.tile_seq = tile_seq;
  ap.tile_q0 = tile_q0;
  ap.order = pair ? pair_order : order;
  ap.cos_t = cos_t;
  ap.sin_t = sin_t;
  ap.out = static_cast<bf16*>(out);
  ap.item_counter = item_counter;
  ap.q_off = nullptr;
  ap.n_blocks = cap;
  ap.H = H;
  ap.Tpad = (int)L.Tpad;
  ap.max_pos = max_pos;
  ap.interleaved = d->rope_interleaved;
  ap.scale_log2 = d->softmax_scale * 1.4426950408889634f;
  if (pair) {
    // persistent grid: one CTA per SM, at most one per work item (blocks of
    // two tiles: sum over sequences of ceil(tiles / 2) <= (tiles + nseq) / 2)
    const int64_t tiles_ub = (T_tot + 127) / 128 + num_seqs;
    int64_t blocks = (tiles_ub + num_seqs) / 2;
    if (blocks > L.cap) blocks = L.cap;
    int64_t grid = blocks * H;
    if (grid > num_sms()) grid = num_sms();
    return launch_attention_pair(N, V, (unsigned)grid, map_q, map_qr, map_kn, map_kr, map_vt, ap, st);
  }
  const unsigned grid = (unsigned)(cap * H);
  return launch_attention_tc(N, V, grid, map_q, map_qr, map_kn, map_kr, map_vt, ap, st);
}

template <typename T>
int launch_decode(const mla_dims* d, const void* q, const void* cache, int64_t cache_num_rows,
                  const int64_t* offsets, const int32_t* lens, const int32_t* positions, int B,
                  int max_len, const void* w_kvb, const float* cos_t, const float* sin_t, int max_pos,
                  void* out, void* workspace, cudaStream_t st) {
  using namespace mla::simt;
  const int H = d->num_heads, R = d->kv_lora_rank, N = d->qk_nope, P = d->qk_rope, V = d->v_head;
  const DecodeWs L = decode_ws_layout(d, B, max_len, false);
  char* ws = static_cast<char*>(workspace);
  float* q_lat = reinterpret_cast<float*>(ws + L.q_lat);
  float* q_rot = reinterpret_cast<float*>(ws + L.q_rot);
  float* o_part = reinterpret_cast<float*>(ws + L.o_part);
  float* m_part = reinterpret_cast<float*>(ws + L.m_part);
  float* l_part = reinterpret_cast<float*>(ws + L.l_part);
  prof_begin(st, "simt_decode_qprep");
  qprep_kernel<T><<<dim3(B, H), 256, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(w_kvb),
                                              positions, cos_t, sin_t, max_pos, H, R, N, P, V,
                                              d->rope_interleaved, q_lat, q_rot);
  prof_end(st);
  const size_t smem = split_smem_bytes(R, P);
  cudaError_t e = cudaFuncSetAttribute(split_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return cuda_status(e, "decode smem attribute");
  dim3 g2(L.nsplit, B, (H + kDecHeads - 1) / kDecHeads);
  prof_begin(st, "simt_decode_split");
  split_kernel<T><<<g2, 256, smem, st>>>(q_lat, q_rot, static_cast<const T*>(cache), cache_num_rows, offsets,
                                         lens, max_len, H, R, P, d->softmax_scale, L.nsplit, o_part, m_part,
                                         l_part);
  prof_end(st);
  prof_begin(st, "simt_decode_combine");
  combine_kernel<T><<<dim3(B, H), 256, 0, st>>>(o_part, m_part, l_part, static_cast<const T*>(w_kvb), H,
                                                R, N, V, L.nsplit, static_cast<T*>(out));
  prof_end(st);
  return cuda_status(cudaGetLastError(), "decode launch");
}

// Tensor-core decode: split schedule -> q absorb + rope -> split-KV attention
// (tcgen05) -> log-sum-exp combine -> W_UV un-absorb.
int launch_decode_tc(const mla_dims* d, const void* q, const void* cache, int64_t cache_rows,
                     const int64_t* offsets, const int32_t* lens, const int32_t* positions, int B, int max_len,
                     const void* w_kvb, const float* cos_t, const float* sin_t, int max_pos, void* out,
                     void* workspace, cudaStream_t st) {
  using bf16 = __nv_bfloat16;
  namespace T = mla::tc;
  const int H = d->num_heads, R = d->kv_lora_rank, N = d->qk_nope, P = d->qk_rope, V = d->v_head;
  const int Hp = T::kDecHeads;   // the workspace's head count: H padded with zero queries
  const DecodeWs L = decode_ws_layout(d, B, max_len, true);
  char* ws = static_cast<char*>(workspace);
  int64_t* prefix = reinterpret_cast<int64_t*>(ws + L.prefix);
  int64_t* meta = reinterpret_cast<int64_t*>(ws + L.meta);
  bf16* qf = reinterpret_cast<bf16*>(ws + L.qf);
  float* o_part = reinterpret_cast<float*>(ws + L.o_part);
  float* m_part = reinterpret_cast<float*>(ws + L.m_part);
  float* l_part = reinterpret_cast<float*>(ws + L.l_part);
  bf16* o_lat = reinterpret_cast<bf16*>(ws + L.o_lat);

  // The cache rows and the absorbed queries as {64 columns, rows, 9 column
  // blocks}: one box brings a whole [rows x 576] tile, laid out in shared
  // memory as nine [rows x 64] blocks (the layout the score product reads).
  CUtensorMap map_cache, map_q;
  {
    const uint64_t dims[3] = {64, (uint64_t)cache_rows, (uint64_t)T::kDecBoxes};
    const uint64_t strides[2] = {(uint64_t)(R + P) * 2, 128};
    const uint32_t box[3] = {64, (uint32_t)T::kDecRows, (uint32_t)T::kDecBoxes};
    int rc = make_map(&map_cache, cache, 3, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {64, (uint64_t)B * Hp, (uint64_t)T::kDecBoxes};
    const uint64_t strides[2] = {(uint64_t)(R + P) * 2, 128};
    const uint32_t box[3] = {64, (uint32_t)Hp, (uint32_t)T::kDecBoxes};
    int rc = make_map(&map_q, qf, 3, dims, strides, box);
    if (rc) return rc;
  }
  // q_lat[b, h, :] = q_nope[b, h, :] W_UK_h   (W_UK_h = rows j < N of head h: [N, R], R contiguous)
  CUtensorMap map_wk, map_qn, map_wv, map_ol;
  {
    const uint64_t dims[2] = {(uint64_t)R, (uint64_t)H * (N + V)};
    const uint64_t strides[1] = {(uint64_t)R * 2};
    const uint32_t box[2] = {64, 64};
    int rc = make_map(&map_wk, w_kvb, 2, dims, strides, box);
    if (rc) return rc;
    const uint32_t box2[2] = {64, 128};
    rc = make_map(&map_wv, w_kvb, 2, dims, strides, box2);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {(uint64_t)(N + P), (uint64_t)H, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)(N + P) * 2, (uint64_t)H * (N + P) * 2};
    const uint32_t box[3] = {64, 1, 64};
    int rc = make_map(&map_qn, q, 3, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {(uint64_t)R, (uint64_t)Hp, (uint64_t)B};
    const uint64_t strides[2] = {(uint64_t)R * 2, (uint64_t)Hp * R * 2};
    const uint32_t box[3] = {64, 1, 64};
    int rc = make_map(&map_ol, o_lat, 3, dims, strides, box);
    if (rc) return rc;
  }
  cudaError_t e = cudaFuncSetAttribute(T::head_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)T::kHgSmem);
  if (e != cudaSuccess) return cuda_status(e, "head gemm smem attribute");
  e = cudaFuncSetAttribute(T::head_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)T::kHgSmem);
  if (e != cudaSuccess) return cuda_status(e, "head gemm smem attribute");
  {
    if (H < Hp) {   // the padded heads' queries are zero (their scores are zero; their outputs unused)
      e = cudaMemset2DAsync(qf + (size_t)H * (R + P), (size_t)Hp * (R + P) * 2, 0, (size_t)(Hp - H) * (R + P) * 2,
                            (size_t)B, st);
      if (e != cudaSuccess) return cuda_status(e, "decode query padding");
    }
    T::HgParams hp{};
    hp.out = qf;
    hp.out_bs = (int64_t)Hp * (R + P);
    hp.out_hs = R + P;
    hp.qf_heads = Hp;
    hp.B = B;
    hp.Nout = R;
    hp.K = N;
    hp.a_row0 = 0;
    hp.a_hstride = N + V;
    hp.q = static_cast<const bf16*>(q);
    hp.positions = positions;
    hp.cos_t = cos_t;
    hp.sin_t = sin_t;
    hp.max_pos = max_pos;
    hp.N = N;
    hp.interleaved = d->rope_interleaved;
    hp.lens = lens;
    hp.offsets = offsets;
    hp.max_len = max_len;
    hp.G = L.G;
    hp.cache_rows = cache_rows;
    hp.prefix = prefix;
    hp.meta = meta;
    // grid x: the H heads plus one column whose first CTA builds the split schedule
    prof_begin(st, "tc_decode_qprep");
    T::head_gemm_kernel<true><<<dim3(H + 1, R / 128, (B + 63) / 64), 192, T::kHgSmem, st>>>(map_wk, map_qn, hp);
    prof_end(st);
  }

  T::DecParams dp;
  dp.prefix = prefix;
  dp.meta = meta;
  dp.offsets = offsets;
  dp.o_part = o_part;
  dp.m_part = m_part;
  dp.l_part = l_part;
  dp.B = B;
  dp.H = Hp;
  dp.R = R;
  dp.scale_log2 = d->softmax_scale * 1.4426950408889634f;
  e = cudaFuncSetAttribute(T::decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)T::kDecSmem);
  if (e != cudaSuccess) return cuda_status(e, "decode smem attribute");
  prof_begin(st, "tc_decode_attention");
  e = launch_dependent(T::decode_attn_kernel, dim3(L.G), dim3(T::kDecThreads), T::kDecSmem, st, map_cache, map_q, dp);
  prof_end(st);
  if (e != cudaSuccess) return cuda_status(e, "decode attention launch");

  prof_begin(st, "tc_decode_combine");
  e = launch_dependent(T::decode_combine_kernel, dim3(B, (H + 3) / 4), dim3(256), 0, st, (const float*)o_part,
                       (const float*)m_part, (const float*)l_part, (const int64_t*)prefix, (const int64_t*)meta, Hp, R,
                       o_lat);
  prof_end(st);
  if (e != cudaSuccess) return cuda_status(e, "decode combine launch");

  // out[b, h, :] = W_UV_h o_lat[b, h, :]   (W_UV_h = rows N .. N+V-1 of head h: [V, R], R contiguous)
  {
    T::HgParams hp{};
    hp.out = static_cast<bf16*>(out);
    hp.out_bs = (int64_t)H * V;
    hp.out_hs = V;
    hp.B = B;
    hp.Nout = V;
    hp.K = R;
    hp.a_row0 = N;
    hp.a_hstride = N + V;
    prof_begin(st, "tc_decode_unabsorb");
    e = launch_dependent(T::head_gemm_kernel<false>, dim3(H, (V + 127) / 128, (B + 63) / 64), dim3(192), T::kHgSmem,
                         st, map_wv, map_ol, hp);
    prof_end(st);
    if (e != cudaSuccess) return cuda_status(e, "decode un-absorb launch");
  }
  return cuda_status(cudaGetLastError(), "decode launch");
}

}  // namespace

extern "C" {

int mla_version(void) { return 100; }

uint64_t mla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int mla_set_kernel_events(void* const* events, int32_t pairs) {
  if (pairs < 0) return fail(MLA_ERR_INVALID_ARG, "pairs must be >= 0");
  g_events = (pairs > 0 && events) ? reinterpret_cast<cudaEvent_t const*>(events) : nullptr;
  g_event_pairs = g_events ? pairs : 0;
  g_event_next = 0;
  return MLA_OK;
}

const char* mla_recorded_kernel_name(int32_t i) {
  if (i < 0 || i >= g_event_next || i >= kMaxNamed) return "";
  return g_event_names[i];
}

int mla_recorded_kernel_events(int32_t* recorded) {
  if (!recorded) return fail(MLA_ERR_INVALID_ARG, "recorded is NULL");
  *recorded = g_event_next;
  return MLA_OK;
}

const char* mla_last_error_string(void) { return g_err; }

const char* mla_last_dispatch(void) { return g_dispatch; }

int mla_softmax_scale(const mla_rope_cfg* rope, int32_t qk_head_dim, float* scale_out) {
  int rc = check_rope(rope);
  if (rc) return rc;
  if (qk_head_dim < 1) return fail(MLA_ERR_INVALID_ARG, "qk_head_dim must be >= 1");
  if (!scale_out) return fail(MLA_ERR_INVALID_ARG, "scale_out is NULL");
  double s = pow((double)qk_head_dim, -0.5);
  if (rope->yarn && rope->mscale_all_dim != 0.0) {
    const double m = yarn_mscale(rope->factor, rope->mscale_all_dim);
    s *= m * m;
  }
  *scale_out = (float)s;
  return MLA_OK;
}

int mla_init_rope_tables(const mla_rope_cfg* rope, int32_t max_pos, float* cos_table,
                         float* sin_table, cudaStream_t stream) {
  int rc = check_rope(rope);
  if (rc) return rc;
  if (max_pos < 1) return fail(MLA_ERR_INVALID_ARG, "max_pos must be >= 1");
  if (!cos_table || !sin_table) return fail(MLA_ERR_INVALID_ARG, "table pointer is NULL");
  mla::RopeTableParams p;
  p.pairs = rope->rope_dim / 2;
  p.rope_dim = rope->rope_dim;
  p.yarn = rope->yarn;
  p.base = rope->base;
  p.factor = rope->factor;
  p.ramp_lo = 0.0;
  p.ramp_hi = 1.0;
  p.table_mscale = 1.0;
  if (rope->yarn) {
    const int dim = rope->rope_dim;
    double lo = floor(correction_dim(rope->beta_fast, dim, rope->base, rope->original_max_pos));
    double hi = ceil(correction_dim(rope->beta_slow, dim, rope->base, rope->original_max_pos));
    if (lo < 0.0) lo = 0.0;
    if (hi > dim - 1) hi = dim - 1;
    if (lo == hi) hi += 0.001;   // the ramp's singular case
    p.ramp_lo = lo;
    p.ramp_hi = hi;
    p.table_mscale = yarn_mscale(rope->factor, rope->mscale) / yarn_mscale(rope->factor, rope->mscale_all_dim);
  }
  const int64_t n = (int64_t)max_pos * p.pairs;
  prof_begin(stream, "rope_tables");
  mla::rope_tables_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(p, max_pos, cos_table, sin_table);
  prof_end(stream);
  return cuda_status(cudaGetLastError(), "rope table launch");
}

int mla_prefill_workspace_size(const mla_dims* dims, int64_t total_tokens, int32_t num_seqs,
                               size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (total_tokens < 0 || num_seqs < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = prefill_ws_bytes(dims, total_tokens, num_seqs);
  return MLA_OK;
}

}  // extern "C"

namespace {
// Bytes of the prepared kv_b_proj copy: fp16 for the tensor-core prefill's
// head shapes, otherwise the weight itself in the run dtype.
size_t prepared_bytes(const mla_dims* d) {
  const size_t n = (size_t)d->num_heads * (d->qk_nope + d->v_head) * d->kv_lora_rank;
  return prefill_tc_shape(d) ? 2 * n : elem_size(d) * n;
}

// mla_prefill (prepared false: w is kv_b_proj, converted on every call) and
// mla_prefill_prepared (prepared true: w comes from mla_prepare_kv_b_proj).
int prefill_entry(const mla_dims* dims, const void* latent, const void* q, const void* w, bool prepared,
                  const void* w_norm, const int32_t* positions, const int32_t* cu_seqlens, int32_t num_seqs,
                  int32_t max_seqlen, int64_t total_tokens, const float* cos_table, const float* sin_table,
                  int32_t max_pos, void* out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0 || max_pos < 1)
    return fail(MLA_ERR_INVALID_ARG, "negative size or max_pos < 1");
  if (num_seqs > 65535) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "num_seqs must be <= 65535");
  if (total_tokens > (int64_t)1 << 31) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "total_tokens too large");
  if (max_seqlen > total_tokens) return fail(MLA_ERR_INVALID_ARG, "max_seqlen exceeds total_tokens");
  if (!cu_seqlens) return fail(MLA_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (total_tokens == 0 || num_seqs == 0 || max_seqlen == 0) return MLA_OK;   // nothing to attend
  if (!latent || !q || !w || !w_norm || !positions || !cos_table || !sin_table || !out)
    return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  const size_t need = prefill_ws_bytes(dims, total_tokens, num_seqs);
  if (!workspace || workspace_bytes < need)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  // (the attention writes each output row with 32-byte stores)
  const bool aligned = aligned16(latent) && aligned16(q) && aligned16(workspace) && aligned16(w_norm) &&
                       aligned16(w) && aligned32(out);
  if (prefill_tc_shape(dims)) {
    if (aligned) {
      set_dispatch("tensor-core");
      return launch_prefill_tc(dims, latent, q, prepared ? nullptr : w, prepared ? w : nullptr, w_norm, positions,
                               cu_seqlens, num_seqs, max_seqlen, total_tokens, cos_table, sin_table, max_pos, out,
                               workspace, stream);
    }
    if (prepared)
      return fail(MLA_ERR_INVALID_ARG,
                  "mla_prefill_prepared needs 16-byte aligned tensors and workspace and a 32-byte aligned out");
    set_dispatch("simt: a tensor or the workspace is not 16-byte aligned, or out not 32-byte aligned");
  } else {
    set_dispatch("simt: head shape or dtype outside the tensor-core kernels");
  }
  // (the prepared copy of a shape outside the tensor-core kernels is the weight itself)
  if (dims->dtype == MLA_FP32)
    return launch_prefill<float>(dims, latent, q, w, w_norm, positions, cu_seqlens, num_seqs,
                                 max_seqlen, total_tokens, cos_table, sin_table, max_pos, out, workspace,
                                 stream);
  return launch_prefill<__nv_bfloat16>(dims, latent, q, w, w_norm, positions, cu_seqlens, num_seqs,
                                       max_seqlen, total_tokens, cos_table, sin_table, max_pos, out,
                                       workspace, stream);
}
}  // namespace

extern "C" {

int mla_prefill(const mla_dims* dims, const void* latent, const void* q, const void* w_kvb,
                const void* w_norm, const int32_t* positions, const int32_t* cu_seqlens,
                int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens, const float* cos_table,
                const float* sin_table, int32_t max_pos, void* out, void* workspace,
                size_t workspace_bytes, cudaStream_t stream) {
  return prefill_entry(dims, latent, q, w_kvb, false, w_norm, positions, cu_seqlens, num_seqs, max_seqlen,
                       total_tokens, cos_table, sin_table, max_pos, out, workspace, workspace_bytes, stream);
}

int mla_kv_b_proj_prepared_size(const mla_dims* dims, size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = prepared_bytes(dims);
  return MLA_OK;
}

int mla_prepare_kv_b_proj(const mla_dims* dims, const void* w_kvb, void* prepared, size_t prepared_bytes_given,
                          cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (!w_kvb || !prepared) return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  const size_t need = prepared_bytes(dims);
  if (prepared_bytes_given < need)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "the prepared weight needs %zu bytes, got %zu", need,
                prepared_bytes_given);
  if (!prefill_tc_shape(dims)) {
    prof_begin(stream, "prepare_kv_b_proj_copy");
    cudaError_t e = cudaMemcpyAsync(prepared, w_kvb, need, cudaMemcpyDeviceToDevice, stream);
    prof_end(stream);
    return cuda_status(e, "prepared weight copy");
  }
  if (!aligned16(w_kvb) || !aligned16(prepared))
    return fail(MLA_ERR_INVALID_ARG, "w_kvb and the prepared buffer must be 16-byte aligned");
  const int64_t n8 = (int64_t)dims->num_heads * (dims->qk_nope + dims->v_head) * dims->kv_lora_rank / 8;
  const int64_t per_block = (int64_t)mla::tc::kPrepThreads * mla::tc::kPrepUnroll;
  prof_begin(stream, "prepare_kv_b_proj");
  mla::tc::weight_f16_kernel<<<(unsigned)((n8 + per_block - 1) / per_block), mla::tc::kPrepThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(w_kvb), static_cast<__half*>(prepared), n8);
  prof_end(stream);
  return cuda_status(cudaGetLastError(), "prepare kv_b_proj launch");
}

int mla_prefill_prepared(const mla_dims* dims, const void* latent, const void* q, const void* w_prepared,
                         const void* w_norm, const int32_t* positions, const int32_t* cu_seqlens,
                         int32_t num_seqs, int32_t max_seqlen, int64_t total_tokens, const float* cos_table,
                         const float* sin_table, int32_t max_pos, void* out, void* workspace,
                         size_t workspace_bytes, cudaStream_t stream) {
  return prefill_entry(dims, latent, q, w_prepared, true, w_norm, positions, cu_seqlens, num_seqs, max_seqlen,
                       total_tokens, cos_table, sin_table, max_pos, out, workspace, workspace_bytes, stream);
}

int mla_decode_workspace_size(const mla_dims* dims, int32_t batch, int32_t max_cache_len, size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (batch < 0 || max_cache_len < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = decode_ws_bytes(dims, batch, max_cache_len);
  return MLA_OK;
}

int mla_decode(const mla_dims* dims, const void* q, const void* cache, int64_t cache_num_rows,
               const int64_t* cache_offsets,
               const int32_t* cache_lens, const int32_t* positions, int32_t batch,
               int32_t max_cache_len, const void* w_kvb, const float* cos_table,
               const float* sin_table, int32_t max_pos, void* out, void* workspace,
               size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (batch < 0) return fail(MLA_ERR_INVALID_ARG, "batch must be >= 0");
  if (batch == 0) return MLA_OK;
  if (max_cache_len < 1) return fail(MLA_ERR_INVALID_ARG, "max_cache_len must be >= 1");
  if (max_pos < 1) return fail(MLA_ERR_INVALID_ARG, "max_pos must be >= 1");
  if (batch > 65535) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "batch must be <= 65535");
  if ((max_cache_len + mla::simt::kDecChunk - 1) / mla::simt::kDecChunk > 256)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "max_cache_len must be <= %d", 256 * mla::simt::kDecChunk);
  if (!q || !cache || !cache_offsets || !cache_lens || !positions || !w_kvb || !cos_table || !sin_table ||
      !out)
    return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (dims->qk_nope > 512) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "qk_nope must be <= 512");
  if (cache_num_rows < 1) return fail(MLA_ERR_INVALID_ARG, "cache_num_rows must be >= 1");
  const size_t need = decode_ws_bytes(dims, batch, max_cache_len);
  if (!workspace || workspace_bytes < need)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  if (!decode_tc_shape(dims)) set_dispatch("simt: head shape or dtype outside the tensor-core decode");
  else if (cache_num_rows >= ((int64_t)1 << 31)) set_dispatch("simt: more than 2^31 cache rows");
  else if (!aligned16(cache) || !aligned16(workspace)) set_dispatch("simt: cache or workspace not 16-byte aligned");
  else set_dispatch("tensor-core");
  if (decode_tc_shape(dims) && cache_num_rows < ((int64_t)1 << 31) && aligned16(cache) && aligned16(workspace))
    return launch_decode_tc(dims, q, cache, cache_num_rows, cache_offsets, cache_lens, positions, batch, max_cache_len,
                            w_kvb, cos_table, sin_table, max_pos, out, workspace, stream);
  if (dims->dtype == MLA_FP32)
    return launch_decode<float>(dims, q, cache, cache_num_rows, cache_offsets, cache_lens, positions, batch,
                                max_cache_len, w_kvb, cos_table, sin_table, max_pos, out, workspace, stream);
  return launch_decode<__nv_bfloat16>(dims, q, cache, cache_num_rows, cache_offsets, cache_lens, positions,
                                      batch, max_cache_len, w_kvb, cos_table, sin_table, max_pos, out,
                                      workspace, stream);
}

int mla_cache_append(const mla_dims* dims, const void* latent, const void* w_norm,
                     const int32_t* positions, int64_t n, const float* cos_table, const float* sin_table,
                     int32_t max_pos, void* cache, int64_t cache_num_rows, const int64_t* cache_rows,
                     cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (n < 0) return fail(MLA_ERR_INVALID_ARG, "n must be >= 0");
  if (n == 0) return MLA_OK;
  if (n > 0x7fffffff) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "too many rows");
  if (max_pos < 1) return fail(MLA_ERR_INVALID_ARG, "max_pos must be >= 1");
  if (!latent || !w_norm || !positions || !cos_table || !sin_table || !cache || !cache_rows)
    return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (cache_num_rows < 1) return fail(MLA_ERR_INVALID_ARG, "cache_num_rows must be >= 1");
  using namespace mla::simt;
  const int R = dims->kv_lora_rank, P = dims->qk_rope;
  prof_begin(stream, "simt_cache_append");
  if (dims->dtype == MLA_FP32)
    cache_append_kernel<float><<<(unsigned)n, 256, 0, stream>>>(
        static_cast<const float*>(latent), static_cast<const float*>(w_norm), positions, cos_table, sin_table,
        max_pos, R, P, dims->rope_interleaved, dims->eps, static_cast<float*>(cache), cache_num_rows,
        cache_rows);
  else
    cache_append_kernel<__nv_bfloat16><<<(unsigned)n, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(latent), static_cast<const __nv_bfloat16*>(w_norm), positions,
        cos_table, sin_table, max_pos, R, P, dims->rope_interleaved, dims->eps,
        static_cast<__nv_bfloat16*>(cache), cache_num_rows, cache_rows);
  prof_end(stream);
  return cuda_status(cudaGetLastError(), "cache append launch");
}

// ---- chunks over a cached prefix ------------------------------------------------
// Workspace: the per-token bookkeeping of chunk_rows_kernel, then the decode's own.
namespace {
struct ChunkWs {
  size_t positions, lens, rows, offsets, decode, total;
};

ChunkWs chunk_ws_layout(const mla_dims* d, int64_t n, int max_total_len) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  ChunkWs L;
  size_t o = 0;
  L.positions = o; o = up(o + (size_t)n * 4);
  L.lens = o;      o = up(o + (size_t)n * 4);
  L.rows = o;      o = up(o + (size_t)n * 8);
  L.offsets = o;   o = up(o + (size_t)n * 8);
  L.decode = o;    o = up(o + decode_ws_bytes(d, (int)n, max_total_len));
  L.total = o;
  return L;
}
constexpr int64_t kMaxChunkTokens = 65535;   // the decode's batch limit

// ---- eager form of the chunk call ---------------------------------------------
// Head shapes it takes: those of the transposed-value GEMM and the two-tile
// attention (bf16, qk_rope 64, v_head 128, qk_nope 64 or 128, rank a multiple
// of 64 up to 512).
bool chunk_eager_shape(const mla_dims* d) {
  return d->dtype == MLA_BF16 && d->qk_rope == 64 && d->v_head == 128 && (d->qk_nope == 64 || d->qk_nope == 128) &&
         d->kv_lora_rank % 64 == 0 && d->kv_lora_rank <= 512;
}
// Average chunk length from which the eager form runs (when the workspace
// holds it): below it every chunk token reading its prefix as one absorbed
// decode row costs less than expanding the prefix's keys and values.
constexpr int64_t kChunkEagerMinAvg = 128;

struct ChunkEagerWs {
  int64_t kcap, qcap, Kpad;
  size_t positions, rows, offsets, lens, seq_ok, kseq_tile0, ktile_seq, ktile_k0, qblk_seq, qblk_q0, qorder,
      counter, w16, c16, k_nope, vt, k_rot, q_rope, total;
};
ChunkEagerWs chunk_eager_ws_layout(const mla_dims* d, int64_t n, int nseq, int max_total_len) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  ChunkEagerWs L{};
  L.kcap = (int64_t)nseq * ((max_total_len + 127) / 128);
  L.qcap = n / 256 + nseq;
  L.Kpad = L.kcap * 128;
  const size_t H = d->num_heads, R = d->kv_lora_rank, N = d->qk_nope, V = d->v_head;
  size_t o = 0;
  L.positions = o;  o = up(o + (size_t)n * 4);
  L.rows = o;       o = up(o + (size_t)n * 8);
  L.offsets = o;    o = up(o + (size_t)n * 8);
  L.lens = o;       o = up(o + (size_t)n * 4);
  L.seq_ok = o;     o = up(o + (size_t)nseq * 4);
  L.kseq_tile0 = o; o = up(o + (size_t)(nseq + 1) * 4);
  L.ktile_seq = o;  o = up(o + (size_t)L.kcap * 4);
  L.ktile_k0 = o;   o = up(o + (size_t)L.kcap * 4);
  L.qblk_seq = o;   o = up(o + (size_t)L.qcap * 4);
  L.qblk_q0 = o;    o = up(o + (size_t)L.qcap * 4);
  L.qorder = o;     o = up(o + (size_t)L.qcap * 4);
  L.counter = o;    o = up(o + 4);
  L.w16 = o;        o = up(o + 2 * H * (N + V) * R);
  L.c16 = o;        o = up(o + 2 * (size_t)L.Kpad * R);
  L.k_nope = o;     o = up(o + 2 * H * (size_t)L.Kpad * N);
  L.vt = o;         o = up(o + 2 * H * V * (size_t)L.Kpad);
  L.k_rot = o;      o = up(o + 2 * (size_t)L.Kpad * 64);
  L.q_rope = o;     o = up(o + 2 * (size_t)n * H * 64);
  L.total = o;
  return L;
}
}  // namespace

// ---- projections on either side of the path ----------------------------------
namespace {
constexpr int64_t kMaxProjRows = (int64_t)1 << 20;   // grid limits of the Linear kernels

// bf16 / fp16 Linears with K a multiple of 64, Nout a multiple of 32 and
// 16-byte aligned operands run on tcgen05 (linear_tc_kernel: 128 rows x bn
// features per CTA, optionally split over K); the others on the CUDA cores.
bool linear_tc(const mla_dims* d, const void* x, const void* w, int K) {
  return d->dtype == MLA_BF16 && K % 64 == 0 && aligned16(x) && aligned16(w);
}

// Most K splits of a Linear whose fp32 result is read by a kernel that adds
// the partials (the workspaces hold this many).
constexpr int kMaxLinSplits = 4;

// Product width (bn) and K splits of a tensor-core Linear: the pair with the
// least estimated time, waves of one CTA per SM times a CTA's work (two
// cycles per feature and K stage at the full tensor rate, plus a fixed cost).
struct LinPlan {
  int bn, splits;
};
LinPlan plan_linear(int64_t n, int K, int Nout, int max_splits) {
  const int cands[4] = {128, 192, 224, 256};
  const int ns = K / 64;
  LinPlan best{256, 1};
  double best_cost = 0.0;
  for (int bn : cands)
    for (int sp = 1; sp <= max_splits && sp <= ns; ++sp) {
      const int64_t ctas = (int64_t)((Nout + bn - 1) / bn) * ((n + 127) / 128) * sp;
      const int64_t waves = (ctas + num_sms() - 1) / num_sms();
      const double cost = (double)waves * ((double)((ns + sp - 1) / sp) * 2.0 * bn + 6000.0);
      if (best_cost == 0.0 || cost < best_cost) {
        best_cost = cost;
        best = LinPlan{bn, sp};
      }
    }
  return best;
}

extern "C++" {   // a template: C++ linkage inside the C-ABI block
template <int kBN, bool kF16>
int launch_linear_tc_t(const CUtensorMap& mx, const CUtensorMap& mw, const mla::tc::LinParams& lp, int64_t n,
                       cudaStream_t st) {
  using C = mla::tc::LinCfg<kBN>;
  auto kern = mla::tc::linear_tc_kernel<kBN, kF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (e != cudaSuccess) return cuda_status(e, "linear smem attribute");
  kern<<<dim3((unsigned)((lp.Nout + kBN - 1) / kBN), (unsigned)((n + 127) / 128), (unsigned)lp.splits),
         mla::tc::kLinThreads, C::kSmem, st>>>(mx, mw, lp);
  return cuda_status(cudaGetLastError(), "linear launch");
}
}  // extern "C++"

// out[t, j] = sum_k x[t, k] w[j, k] for x [n, K], w [Nout, K], out [n, Nout]
// (row-major). x and w are in the run dtype, or both fp16 when `f16_operands`;
// the result goes to `out` in the run dtype, or to out_f32 in fp32 when that
// is set. With max_splits > 1 the tensor-core Linear may split K: out_f32
// then holds *splits partials [splits][n][Nout] that the consumer adds in
// split order (*splits is 1 otherwise).
int launch_linear(const mla_dims* d, const void* x, const void* w, void* out, int64_t n, int K, int Nout,
                  cudaStream_t st, const char* name, float* out_f32 = nullptr, bool f16_operands = false,
                  int max_splits = 1, int* splits = nullptr) {
  namespace T = mla::tc;
  if (splits) *splits = 1;
  if (linear_tc(d, x, w, K) && Nout % 32 == 0 && aligned16(out_f32 ? (const void*)out_f32 : out)) {
    const CUtensorMapDataType dt = f16_operands ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const LinPlan pl = plan_linear(n, K, Nout, out_f32 ? max_splits : 1);
    CUtensorMap map_w, map_x;
    {
      const uint64_t dims[2] = {(uint64_t)K, (uint64_t)Nout};
      const uint64_t strides[1] = {(uint64_t)K * 2};
      const uint32_t box[2] = {64, (uint32_t)pl.bn};
      int rc = make_map(&map_w, w, 2, dims, strides, box, dt);
      if (rc) return rc;
    }
    {
      const uint64_t dims[2] = {(uint64_t)K, (uint64_t)n};
      const uint64_t strides[1] = {(uint64_t)K * 2};
      const uint32_t box[2] = {64, 128};
      int rc = make_map(&map_x, x, 2, dims, strides, box, dt);
      if (rc) return rc;
    }
    T::LinParams lp{};
    lp.n = n;
    lp.K = K;
    lp.Nout = Nout;
    lp.splits = pl.splits;
    lp.out = static_cast<__nv_bfloat16*>(out);
    lp.out_f32 = out_f32;
    if (splits) *splits = pl.splits;
    prof_begin(st, name);
    int rc = MLA_OK;
#define MLA_LIN_CASE(c)                                                                     \
    if (pl.bn == c) rc = f16_operands ? launch_linear_tc_t<c, true>(map_x, map_w, lp, n, st) \
                                      : launch_linear_tc_t<c, false>(map_x, map_w, lp, n, st);
    MLA_LIN_CASE(128) MLA_LIN_CASE(192) MLA_LIN_CASE(224) MLA_LIN_CASE(256)
#undef MLA_LIN_CASE
    prof_end(st);
    return rc;
  }
  const dim3 grid((unsigned)((Nout + mla::kLinTile - 1) / mla::kLinTile),
                  (unsigned)((n + mla::kLinTile - 1) / mla::kLinTile));
  using bf16 = __nv_bfloat16;
  prof_begin(st, name);
  if (d->dtype == MLA_FP32)
    mla::simt_linear_kernel<float><<<grid, mla::kLinTile * mla::kLinTile, 0, st>>>(
        static_cast<const float*>(x), static_cast<const float*>(w), static_cast<float*>(out), n, K, Nout);
  else if (out_f32)
    mla::simt_linear_kernel<bf16, bf16, float><<<grid, mla::kLinTile * mla::kLinTile, 0, st>>>(
        static_cast<const bf16*>(x), static_cast<const bf16*>(w), out_f32, n, K, Nout);
  else
    mla::simt_linear_kernel<bf16><<<grid, mla::kLinTile * mla::kLinTile, 0, st>>>(
        static_cast<const bf16*>(x), static_cast<const bf16*>(w), static_cast<bf16*>(out), n, K, Nout);
  prof_end(st);
  return cuda_status(cudaGetLastError(), name);
}

// A CUDA-core Linear whose x is fp32 (the normalized q_a of a bf16 run whose
// q_b_proj cannot take the tensor cores) and whose w and out are bf16.
int launch_linear_f32x(const float* x, const void* w, void* out, int64_t n, int K, int Nout, cudaStream_t st,
                       const char* name) {
  using bf16 = __nv_bfloat16;
  const dim3 grid((unsigned)((Nout + mla::kLinTile - 1) / mla::kLinTile),
                  (unsigned)((n + mla::kLinTile - 1) / mla::kLinTile));
  prof_begin(st, name);
  mla::simt_linear_kernel<float, bf16, bf16><<<grid, mla::kLinTile * mla::kLinTile, 0, st>>>(
      x, static_cast<const bf16*>(w), static_cast<bf16*>(out), n, K, Nout);
  prof_end(st);
  return cuda_status(cudaGetLastError(), name);
}

// Workspace of mla_kv_down_append: the fp32 result of the Linear (bf16 runs),
// room for kMaxLinSplits K-split partials.
size_t kv_down_ws_bytes(const mla_dims* d, int64_t n) {
  return d->dtype == MLA_BF16 ? align_up((size_t)kMaxLinSplits * n * (d->kv_lora_rank + d->qk_rope) * 4, 256) : 0;
}

// Workspace of mla_q_proj. fp32 runs: q_a [n, q_rank] fp32, normalized in
// place. bf16 runs: q_a as up to kMaxLinSplits fp32 partials [n, q_rank], its
// normalized copy [n, q_rank] (fp16 for the tensor-core q_b_proj), and the
// fp16 copy of w_qb.
struct QProjWs {
  size_t q_a, q_an, w16, total;
};
QProjWs q_proj_ws_layout(const mla_dims* d, int32_t q_rank, int64_t n) {
  QProjWs L{};
  size_t off = 0;
  // bf16: q_a_proj's fp32 partials (up to kMaxLinSplits K splits)
  L.q_a = off; off = align_up(off + (size_t)(d->dtype == MLA_BF16 ? kMaxLinSplits : 1) * n * q_rank * 4, 256);
  if (d->dtype == MLA_BF16) {
    L.q_an = off; off = align_up(off + (size_t)n * q_rank * 4, 256);   // fp16 (tensor cores) or fp32 (CUDA cores)
    L.w16 = off;  off = align_up(off + (size_t)d->num_heads * (d->qk_nope + d->qk_rope) * q_rank * 2, 256);
  }
  L.total = off;
  return L;
}

int check_proj_rows(int64_t n) {
  if (n < 0) return fail(MLA_ERR_INVALID_ARG, "n must be >= 0");
  if (n > kMaxProjRows) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "at most %lld rows per call", (long long)kMaxProjRows);
  return MLA_OK;
}

}  // namespace

// Device address of g_noalloc_scratch on the current device. Host code cannot
// use the array's name as a device address, so every call looks the address
// up (a host-side lookup, no stream operation): after a device reset or in a
// new context the array lives at a new address, and a kept pointer would be
// stale. The first lookup on a device may load the library's device code.
namespace {
int noalloc_scratch(void** ptr) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress of the static scratch");
  *ptr = p;
  return MLA_OK;
}
}  // namespace

int mla_prefill_noalloc(const mla_dims* dims, const void* latent, const void* q, const void* w_kvb,
                        const void* w_norm, const int32_t* positions, const int32_t* cu_seqlens, int32_t num_seqs,
                        int32_t max_seqlen, int64_t total_tokens, const float* cos_table, const float* sin_table,
                        int32_t max_pos, void* out, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (total_tokens < 0 || num_seqs < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  const size_t need = prefill_ws_bytes(dims, total_tokens, num_seqs);
  if (need > (size_t)MLA_NOALLOC_SCRATCH_BYTES)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL,
                "this prefill needs %zu bytes of scratch; the static scratch of mla_prefill_noalloc holds %zu",
                need, (size_t)MLA_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  return mla_prefill(dims, latent, q, w_kvb, w_norm, positions, cu_seqlens, num_seqs, max_seqlen, total_tokens,
                     cos_table, sin_table, max_pos, out, scratch, (size_t)MLA_NOALLOC_SCRATCH_BYTES, stream);
}

int mla_prefill_cached_workspace_size(const mla_dims* dims, int64_t total_tokens, int32_t max_total_len,
                                      size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (total_tokens < 0 || max_total_len < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (total_tokens > kMaxChunkTokens)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "at most %lld chunk tokens per call", (long long)kMaxChunkTokens);
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = chunk_ws_layout(dims, total_tokens, max_total_len).total;
  return MLA_OK;
}

}  // extern "C"

namespace {
// The eager form: bookkeeping and append as in the absorbed form, then the
// schedule over key tiles and query blocks, the fp16 weight copy, the padded
// key rows (cached normalized latent and rotated key), zeroed outputs of
// invalid sequences, the up-projection of every key row, and the two-tile
// attention of the chunk's queries with each sequence's prefix length as
// the query offset.
int launch_prefill_cached_eager(const mla_dims* d, const void* latent, const void* q, const void* w_kvb,
                                const void* w_norm, const int32_t* cu_seqlens, int nseq, int64_t Tq,
                                const int64_t* cache_offsets, const int32_t* prefix_lens, int max_total_len,
                                const float* cos_t, const float* sin_t, int max_pos, void* cache,
                                int64_t cache_num_rows, void* out, void* workspace, cudaStream_t st) {
  using bf16 = __nv_bfloat16;
  namespace T = mla::tc;
  const int H = d->num_heads, R = d->kv_lora_rank, N = d->qk_nope, P = d->qk_rope, V = d->v_head;
  const ChunkEagerWs L = chunk_eager_ws_layout(d, Tq, nseq, max_total_len);
  char* ws = static_cast<char*>(workspace);
  int32_t* positions = reinterpret_cast<int32_t*>(ws + L.positions);
  int64_t* rows = reinterpret_cast<int64_t*>(ws + L.rows);
  int64_t* offsets = reinterpret_cast<int64_t*>(ws + L.offsets);
  int32_t* lens = reinterpret_cast<int32_t*>(ws + L.lens);
  int32_t* seq_ok = reinterpret_cast<int32_t*>(ws + L.seq_ok);
  int32_t* kseq_tile0 = reinterpret_cast<int32_t*>(ws + L.kseq_tile0);
  int32_t* ktile_seq = reinterpret_cast<int32_t*>(ws + L.ktile_seq);
  int32_t* ktile_k0 = reinterpret_cast<int32_t*>(ws + L.ktile_k0);
  int32_t* qblk_seq = reinterpret_cast<int32_t*>(ws + L.qblk_seq);
  int32_t* qblk_q0 = reinterpret_cast<int32_t*>(ws + L.qblk_q0);
  int32_t* qorder = reinterpret_cast<int32_t*>(ws + L.qorder);
  int32_t* counter = reinterpret_cast<int32_t*>(ws + L.counter);
  __half* w16 = reinterpret_cast<__half*>(ws + L.w16);
  __half* c16 = reinterpret_cast<__half*>(ws + L.c16);
  __half* k_nope = reinterpret_cast<__half*>(ws + L.k_nope);
  __half* vt = reinterpret_cast<__half*>(ws + L.vt);
  __half* k_rot = reinterpret_cast<__half*>(ws + L.k_rot);
  const int NOUT = H * (N + V);

  // 1. per-token positions and cache rows; 2. the chunk's rows into the cache
  prof_begin(st, "chunk_rows");
  mla::chunk_rows_kernel<<<(unsigned)((Tq + mla::kChunkThreads - 1) / mla::kChunkThreads), mla::kChunkThreads, 0,
                           st>>>(cu_seqlens, nseq, Tq, cache_offsets, prefix_lens, max_total_len, max_pos,
                                 cache_num_rows, positions, rows, offsets, lens);
  prof_end(st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "chunk rows launch");
  int rc = mla_cache_append(d, latent, w_norm, positions, Tq, cos_t, sin_t, max_pos, cache, cache_num_rows, rows,
                            st);
  if (rc) return rc;
  // 3. schedule (one block); 4. fp16 weight copy
  prof_begin(st, "chunk_eager_schedule");
  T::chunk_eager_schedule_kernel<<<1, T::kChunkSchedThreads, 0, st>>>(
      cu_seqlens, nseq, Tq, cache_offsets, prefix_lens, max_total_len, max_pos, cache_num_rows, (int)L.kcap,
      (int)L.qcap, seq_ok, kseq_tile0, ktile_seq, ktile_k0, qblk_seq, qblk_q0, qorder, counter);
  prof_end(st);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "chunk schedule launch");
  const int64_t n8 = (int64_t)NOUT * R / 8;
  const int64_t per_block = (int64_t)T::kPrepThreads * T::kPrepUnroll;
  prof_begin(st, "chunk_weight_f16");
  T::weight_f16_kernel<<<(unsigned)((n8 + per_block - 1) / per_block), T::kPrepThreads, 0, st>>>(
      static_cast<const bf16*>(w_kvb), w16, n8);
  prof_end(st);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "chunk weight launch");
  // 5. padded key rows from the cache; 6. zero outputs of invalid sequences
  prof_begin(st, "chunk_eager_rows");
  e = launch_dependent(T::chunk_eager_rows_kernel, dim3((unsigned)((L.Kpad + T::kChunkRowsPerBlock - 1) /
                                                                    T::kChunkRowsPerBlock)),
                       dim3(32 * T::kChunkRowsPerBlock), 0, st, (const bf16*)cache, R, cache_offsets, prefix_lens,
                       cu_seqlens, (const int32_t*)ktile_seq, (const int32_t*)ktile_k0, (int64_t)L.Kpad, c16, k_rot);
  prof_end(st);
  if (e != cudaSuccess) return cuda_status(e, "chunk key rows launch");
  prof_begin(st, "chunk_eager_zero");
  e = launch_dependent(T::chunk_eager_zero_kernel, dim3((unsigned)((Tq + T::kChunkRowsPerBlock - 1) /
                                                                   T::kChunkRowsPerBlock)),
                       dim3(32 * T::kChunkRowsPerBlock), 0, st, cu_seqlens, nseq, Tq, (const int32_t*)seq_ok, H * V,
                       static_cast<bf16*>(out));
  prof_end(st);
  if (e != cudaSuccess) return cuda_status(e, "chunk zero launch");
  // the queries' rotary parts, turned at their positions (fp16)
  T::QRopeParams qrp{};
  qrp.q = static_cast<const bf16*>(q);
  qrp.positions = positions;
  qrp.cos_t = cos_t;
  qrp.sin_t = sin_t;
  qrp.qr = reinterpret_cast<__half*>(ws + L.q_rope);
  qrp.rows = Tq * H;
  qrp.H = H; qrp.D = N + P; qrp.N = N; qrp.max_pos = max_pos; qrp.interleaved = d->rope_interleaved;
  if (qrp.rows > 0) {
    prof_begin(st, "tc_q_rope");
    e = launch_dependent(T::q_rope_kernel, dim3((unsigned)T::q_rope_blocks(qrp.rows, H, T::kPrepThreads)),
                         dim3(T::kPrepThreads), 0, st, qrp);
    prof_end(st);
    if (e != cudaSuccess) return cuda_status(e, "q rope launch");
  }

  // 7. k_nope / transposed values of every key row
  CUtensorMap map_w, map_c16;
  {
    const uint64_t dims[2] = {(uint64_t)R, (uint64_t)NOUT};
    const uint64_t strides[1] = {(uint64_t)R * 2};
    const uint32_t box[2] = {64, (uint32_t)(N + V)};
    rc = make_map(&map_w, w16, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)R, (uint64_t)L.Kpad};
    const uint64_t strides[1] = {(uint64_t)R * 2};
    const uint32_t box[2] = {64, 128};
    rc = make_map(&map_c16, c16, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  T::GemmParams gp{};
  gp.cu = cu_seqlens;
  gp.tile_seq = ktile_seq;
  gp.tile_q0 = ktile_k0;
  gp.k_nope = k_nope;
  gp.vt = vt;
  gp.k_rot = k_rot;
  gp.Ttot = Tq;
  gp.Tpad = (int)L.Kpad;
  gp.R = R; gp.P = P; gp.H = H; gp.N = N; gp.V = V; gp.NOUT = NOUT;
  gp.max_pos = max_pos;
  gp.interleaved = d->rope_interleaved;
  gp.eps = d->eps;
  gp.a_padded = 1;
  gp.knope_bf16 = 1;
  int groups = num_sms() / (int)(L.kcap > 0 ? L.kcap : 1);
  if (groups < 1) groups = 1;
  if (groups > H) groups = H;
  gp.tiles_per_cta = (H + groups - 1) / groups;
  const int gy = (H + gp.tiles_per_cta - 1) / gp.tiles_per_cta;
  auto gemm = N == 64 ? T::norm_kvb_gemm_vt_kernel<64> : T::norm_kvb_gemm_vt_kernel<128>;
  e = cudaFuncSetAttribute(gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)T::kG2SmemBytes);
  if (e != cudaSuccess) return cuda_status(e, "gemm smem attribute");
  prof_begin(st, "tc_norm_kv_b_proj");
  e = launch_dependent(gemm, dim3((unsigned)L.kcap, (unsigned)gy), dim3(T::kG2Threads), T::kG2SmemBytes, st, map_c16,
                       map_w, gp);
  prof_end(st);
  if (e != cudaSuccess) return cuda_status(e, "gemm launch");

  // 8. the chunk's queries against each sequence's keys
  const int D = N + P;
  CUtensorMap map_q, map_qr, map_kn, map_kr, map_vt;
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)H, (uint64_t)Tq};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)H * D * 2};
    const uint32_t box[3] = {64, 1, 128};
    rc = make_map(&map_q, q, 3, dims, strides, box);
    if (rc) return rc;
  }
  {
    const uint64_t dims[3] = {(uint64_t)P, (uint64_t)H, (uint64_t)Tq};
    const uint64_t strides[2] = {(uint64_t)P * 2, (uint64_t)H * P * 2};
    const uint32_t box[3] = {64, 1, 128};
    rc = make_map(&map_qr, ws + L.q_rope, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)N, (uint64_t)H * L.Kpad};
    const uint64_t strides[1] = {(uint64_t)N * 2};
    const uint32_t box[2] = {64, (uint32_t)T::kPrBKV};
    rc = make_map(&map_kn, k_nope, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)P, (uint64_t)L.Kpad};
    const uint64_t strides[1] = {(uint64_t)P * 2};
    const uint32_t box[2] = {64, (uint32_t)T::kPrBKV};
    rc = make_map(&map_kr, k_rot, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)L.Kpad, (uint64_t)H * V};
    const uint64_t strides[1] = {(uint64_t)L.Kpad * 2};
    const uint32_t box[2] = {64, (uint32_t)V};
    rc = make_map(&map_vt, vt, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
    if (rc) return rc;
  }
  T::AttParams ap{};
  ap.cu = cu_seqlens;
  ap.positions = positions;
  ap.seq_tile0 = kseq_tile0;
  ap.tile_seq = qblk_seq;
  ap.tile_q0 = qblk_q0;
  ap.order = qorder;
  ap.cos_t = cos_t;
  ap.sin_t = sin_t;
  ap.out = static_cast<bf16*>(out);
  ap.item_counter = counter;
  ap.q_off = prefix_lens;
  ap.n_blocks = (int)L.qcap;
  ap.H = H;
  ap.Tpad = (int)L.Kpad;
  ap.max_pos = max_pos;
  ap.interleaved = d->rope_interleaved;
  ap.scale_log2 = d->softmax_scale * 1.4426950408889634f;
  int64_t grid = L.qcap * H;
  if (grid > num_sms()) grid = num_sms();
  return launch_attention_pair(N, V, (unsigned)grid, map_q, map_qr, map_kn, map_kr, map_vt, ap, st);
}
}  // namespace

extern "C" {

int mla_prefill_cached_eager_workspace_size(const mla_dims* dims, int64_t total_tokens, int32_t num_seqs,
                                            int32_t max_total_len, size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  if (total_tokens < 0 || num_seqs < 0 || max_total_len < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (total_tokens > kMaxChunkTokens)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "at most %lld chunk tokens per call", (long long)kMaxChunkTokens);
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  if (!chunk_eager_shape(dims)) return fail(MLA_ERR_UNSUPPORTED_SHAPE, "no eager chunk form for this head shape");
  if ((int64_t)num_seqs * ((max_total_len + 127) / 128) > 0x7fffffff / 128)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "too many key rows for the eager chunk form");
  *bytes = chunk_eager_ws_layout(dims, total_tokens, num_seqs, max_total_len).total;
  return MLA_OK;
}

int mla_prefill_cached(const mla_dims* dims, const void* latent, const void* q, const void* w_kvb,
                       const void* w_norm, const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                       const int64_t* cache_offsets, const int32_t* prefix_lens, int32_t max_total_len,
                       const float* cos_table, const float* sin_table, int32_t max_pos, void* cache,
                       int64_t cache_num_rows, void* out, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  return mla_prefill_cached_form(dims, latent, q, w_kvb, w_norm, cu_seqlens, num_seqs, total_tokens, cache_offsets,
                                 prefix_lens, max_total_len, cos_table, sin_table, max_pos, cache, cache_num_rows, out,
                                 workspace, workspace_bytes, MLA_CHUNK_AUTO, stream);
}

int mla_prefill_cached_form(const mla_dims* dims, const void* latent, const void* q, const void* w_kvb,
                            const void* w_norm, const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                            const int64_t* cache_offsets, const int32_t* prefix_lens, int32_t max_total_len,
                            const float* cos_table, const float* sin_table, int32_t max_pos, void* cache,
                            int64_t cache_num_rows, void* out, void* workspace, size_t workspace_bytes,
                            int32_t form, cudaStream_t stream) {
  if (form != MLA_CHUNK_AUTO && form != MLA_CHUNK_ABSORBED && form != MLA_CHUNK_EAGER)
    return fail(MLA_ERR_INVALID_ARG, "form must be MLA_CHUNK_AUTO, MLA_CHUNK_ABSORBED or MLA_CHUNK_EAGER");
  int rc = check_dims(dims);
  if (rc) return rc;
  if (total_tokens < 0 || num_seqs < 0) return fail(MLA_ERR_INVALID_ARG, "negative size");
  if (total_tokens == 0) return MLA_OK;
  if (num_seqs < 1) return fail(MLA_ERR_INVALID_ARG, "num_seqs must be >= 1 when there are chunk tokens");
  if (total_tokens > kMaxChunkTokens)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "at most %lld chunk tokens per call", (long long)kMaxChunkTokens);
  if (max_total_len < 1) return fail(MLA_ERR_INVALID_ARG, "max_total_len must be >= 1");
  // the decode's own limit, checked here so that nothing is written to the cache first
  if ((max_total_len + mla::simt::kDecChunk - 1) / mla::simt::kDecChunk > 256)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "max_total_len must be <= %d", 256 * mla::simt::kDecChunk);
  if (max_pos < 1) return fail(MLA_ERR_INVALID_ARG, "max_pos must be >= 1");
  if (cache_num_rows < 1) return fail(MLA_ERR_INVALID_ARG, "cache_num_rows must be >= 1");
  if (!latent || !q || !w_kvb || !w_norm || !cu_seqlens || !cache_offsets || !prefix_lens || !cos_table ||
      !sin_table || !cache || !out)
    return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  // automatic: long chunks (on average kChunkEagerMinAvg tokens or more per
  // sequence) take the eager form when the workspace holds it
  const bool eager_ok = chunk_eager_shape(dims) && aligned16(q) && aligned16(cache) && aligned16(w_kvb) &&
                        aligned32(out) && aligned16(workspace) &&
                        (int64_t)num_seqs * ((max_total_len + 127) / 128) <= 0x7fffffff / 128;
  if (form == MLA_CHUNK_EAGER && !eager_ok)
    return fail(MLA_ERR_UNSUPPORTED_SHAPE, "the eager form needs the tensor-core head shapes and 16-byte alignment");
  if (form == MLA_CHUNK_EAGER ||
      (form == MLA_CHUNK_AUTO && eager_ok && total_tokens >= kChunkEagerMinAvg * num_seqs)) {
    const size_t need_eager = chunk_eager_ws_layout(dims, total_tokens, num_seqs, max_total_len).total;
    if (form == MLA_CHUNK_EAGER && (!workspace || workspace_bytes < need_eager))
      return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "the eager form needs %zu bytes of workspace, got %zu", need_eager,
                  workspace_bytes);
    if (workspace && workspace_bytes >= need_eager) {
      set_dispatch("eager: keys and values of every cached row expanded, two-tile attention");
      return launch_prefill_cached_eager(dims, latent, q, w_kvb, w_norm, cu_seqlens, num_seqs, total_tokens,
                                         cache_offsets, prefix_lens, max_total_len, cos_table, sin_table, max_pos,
                                         cache, cache_num_rows, out, workspace, stream);
    }
  }
  const ChunkWs L = chunk_ws_layout(dims, total_tokens, max_total_len);
  if (!workspace || workspace_bytes < L.total)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", L.total, workspace_bytes);
  char* ws = static_cast<char*>(workspace);
  int32_t* positions = reinterpret_cast<int32_t*>(ws + L.positions);
  int32_t* lens = reinterpret_cast<int32_t*>(ws + L.lens);
  int64_t* rows = reinterpret_cast<int64_t*>(ws + L.rows);
  int64_t* offsets = reinterpret_cast<int64_t*>(ws + L.offsets);
  prof_begin(stream, "chunk_rows");
  mla::chunk_rows_kernel<<<(unsigned)((total_tokens + mla::kChunkThreads - 1) / mla::kChunkThreads),
                           mla::kChunkThreads, 0, stream>>>(cu_seqlens, num_seqs, total_tokens, cache_offsets,
                                                            prefix_lens, max_total_len, max_pos, cache_num_rows,
                                                            positions, rows, offsets, lens);
  prof_end(stream);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "chunk rows launch");
  // 1. the chunk's rows go into the cache; 2. each chunk token attends to its
  // sequence's rows up to and including its own, as one absorbed decode row
  rc = mla_cache_append(dims, latent, w_norm, positions, total_tokens, cos_table, sin_table, max_pos, cache,
                        cache_num_rows, rows, stream);
  if (rc) return rc;
  rc = mla_decode(dims, q, cache, cache_num_rows, offsets, lens, positions, (int32_t)total_tokens, max_total_len,
                  w_kvb, cos_table, sin_table, max_pos, out, ws + L.decode, workspace_bytes - L.decode, stream);
  if (!rc) set_dispatch(strcmp(g_dispatch, "tensor-core") == 0 ? "absorbed: one tensor-core decode row per chunk token"
                                                               : "absorbed: one CUDA-core decode row per chunk token");
  return rc;
}

int mla_kv_down_append_workspace_size(const mla_dims* dims, int64_t n, size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_proj_rows(n);
  if (rc) return rc;
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = kv_down_ws_bytes(dims, n);
  return MLA_OK;
}

int mla_kv_down_append(const mla_dims* dims, int32_t hidden_size, const void* hidden, const void* w_kva,
                       const void* w_norm, const int32_t* positions, int64_t n, const float* cos_table,
                       const float* sin_table, int32_t max_pos, void* latent, void* cache, int64_t cache_num_rows,
                       const int64_t* cache_rows, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_proj_rows(n);
  if (rc) return rc;
  if (hidden_size < 1) return fail(MLA_ERR_INVALID_ARG, "hidden_size must be >= 1");
  if (!hidden || !w_kva || !latent) return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  const bool append = cache != nullptr || cache_rows != nullptr;
  if (append && (!cache || !cache_rows || !w_norm || !positions || !cos_table || !sin_table))
    return fail(MLA_ERR_INVALID_ARG, "appending needs cache, cache_rows, w_norm, positions and the tables");
  if (append && (max_pos < 1 || cache_num_rows < 1))
    return fail(MLA_ERR_INVALID_ARG, "appending needs max_pos >= 1 and cache_num_rows >= 1");
  if (n == 0) return MLA_OK;
  const size_t need = kv_down_ws_bytes(dims, n);
  if (need && (!workspace || workspace_bytes < need))
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", need, workspace_bytes);
  const int W = dims->kv_lora_rank + dims->qk_rope;
  if (dims->dtype == MLA_FP32) {
    rc = launch_linear(dims, hidden, w_kva, latent, n, hidden_size, W, stream, "kv_a_proj");
    if (rc || !append) return rc;
    return mla_cache_append(dims, latent, w_norm, positions, n, cos_table, sin_table, max_pos, cache,
                            cache_num_rows, cache_rows, stream);
  }
  // bf16: the Linear's fp32 result, then compressed_kv and the cache row from it
  float* x32 = static_cast<float*>(workspace);
  int splits = 1;
  rc = launch_linear(dims, hidden, w_kva, nullptr, n, hidden_size, W, stream, "kv_a_proj", x32, false,
                     kMaxLinSplits, &splits);
  if (rc) return rc;
  prof_begin(stream, "kv_latent_append");
  cudaError_t e = launch_dependent(
      mla::kv_latent_append_kernel, dim3((unsigned)((n + mla::kKvRowsPerBlock - 1) / mla::kKvRowsPerBlock)),
      dim3(32 * mla::kKvRowsPerBlock), 0, stream, (const float*)x32, splits, (int64_t)(n * W),
      static_cast<__nv_bfloat16*>(latent), n, dims->kv_lora_rank, dims->qk_rope,
      static_cast<const __nv_bfloat16*>(w_norm), positions, cos_table, sin_table, max_pos, dims->rope_interleaved,
      dims->eps, append ? static_cast<__nv_bfloat16*>(cache) : (__nv_bfloat16*)nullptr, cache_num_rows, cache_rows);
  prof_end(stream);
  if (e != cudaSuccess) return cuda_status(e, "kv latent append launch");
  return cuda_status(cudaGetLastError(), "kv latent append launch");
}

int mla_q_proj_workspace_size(const mla_dims* dims, int32_t q_rank, int64_t n, size_t* bytes) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_proj_rows(n);
  if (rc) return rc;
  if (q_rank < 1) return fail(MLA_ERR_INVALID_ARG, "q_rank must be >= 1");
  if (!bytes) return fail(MLA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = q_proj_ws_layout(dims, q_rank, n).total;
  return MLA_OK;
}

int mla_q_proj(const mla_dims* dims, int32_t hidden_size, int32_t q_rank, const void* hidden, const void* w_qa,
               const void* w_qnorm, const void* w_qb, int64_t n, void* q, void* workspace, size_t workspace_bytes,
               cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_proj_rows(n);
  if (rc) return rc;
  if (hidden_size < 1 || q_rank < 1) return fail(MLA_ERR_INVALID_ARG, "hidden_size and q_rank must be >= 1");
  if (!hidden || !w_qa || !w_qnorm || !w_qb || !q) return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (n == 0) return MLA_OK;
  const QProjWs L = q_proj_ws_layout(dims, q_rank, n);
  if (!workspace || workspace_bytes < L.total)
    return fail(MLA_ERR_WORKSPACE_TOO_SMALL, "workspace needs %zu bytes, got %zu", L.total, workspace_bytes);
  char* ws = static_cast<char*>(workspace);
  const int NQ = dims->num_heads * (dims->qk_nope + dims->qk_rope);
  const unsigned blocks = (unsigned)((n + mla::kRowsPerNormBlock - 1) / mla::kRowsPerNormBlock);
  if (dims->dtype == MLA_FP32) {
    // q_a = hidden W_qa^T, normalized in place, then q = q_a W_qb^T
    float* qa = reinterpret_cast<float*>(ws + L.q_a);
    rc = launch_linear(dims, hidden, w_qa, qa, n, hidden_size, q_rank, stream, "q_a_proj");
    if (rc) return rc;
    prof_begin(stream, "q_a_layernorm");
    mla::rmsnorm_rows_kernel<float><<<blocks, 32 * mla::kRowsPerNormBlock, 0, stream>>>(
        qa, static_cast<const float*>(w_qnorm), qa, n, q_rank, dims->eps);
    prof_end(stream);
    rc = cuda_status(cudaGetLastError(), "q_a_layernorm launch");
    if (rc) return rc;
    return launch_linear(dims, qa, w_qb, q, n, q_rank, NQ, stream, "q_b_proj");
  }
  // bf16: q_a_proj's fp32 result is normalized without a rounding in between;
  // the normalized q_a feeds q_b_proj in fp16 against an fp16 copy of w_qb
  // (tensor cores), or in fp32 (CUDA cores)
  float* qa32 = reinterpret_cast<float*>(ws + L.q_a);
  int splits = 1;
  rc = launch_linear(dims, hidden, w_qa, nullptr, n, hidden_size, q_rank, stream, "q_a_proj", qa32, false,
                     kMaxLinSplits, &splits);
  if (rc) return rc;
  const bool tc_b = linear_tc(dims, ws + L.q_an, w_qb, q_rank) && aligned16(q);
  if (tc_b) {
    __half* qan = reinterpret_cast<__half*>(ws + L.q_an);
    __half* w16 = reinterpret_cast<__half*>(ws + L.w16);
    const int64_t n8 = (int64_t)NQ * q_rank / 8;
    const int64_t per_block = (int64_t)mla::tc::kPrepThreads * mla::tc::kPrepUnroll;
    if ((int64_t)NQ * q_rank % 8 == 0) {
      prof_begin(stream, "q_b_proj_weight_f16");
      mla::tc::weight_f16_kernel<<<(unsigned)((n8 + per_block - 1) / per_block), mla::tc::kPrepThreads, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(w_qb), w16, n8);
      prof_end(stream);
      rc = cuda_status(cudaGetLastError(), "q_b_proj weight launch");
      if (rc) return rc;
      prof_begin(stream, "q_a_layernorm");
      mla::rmsnorm_f32_rows_kernel<__half><<<blocks, 32 * mla::kRowsPerNormBlock, 0, stream>>>(
          qa32, splits, n * q_rank, static_cast<const __nv_bfloat16*>(w_qnorm), qan, n, q_rank, dims->eps);
      prof_end(stream);
      rc = cuda_status(cudaGetLastError(), "q_a_layernorm launch");
      if (rc) return rc;
      return launch_linear(dims, qan, w16, q, n, q_rank, NQ, stream, "q_b_proj", nullptr, true);
    }
  }
  float* qan32 = reinterpret_cast<float*>(ws + L.q_an);
  prof_begin(stream, "q_a_layernorm");
  mla::rmsnorm_f32_rows_kernel<float><<<blocks, 32 * mla::kRowsPerNormBlock, 0, stream>>>(
      qa32, splits, n * q_rank, static_cast<const __nv_bfloat16*>(w_qnorm), qan32, n, q_rank, dims->eps);
  prof_end(stream);
  rc = cuda_status(cudaGetLastError(), "q_a_layernorm launch");
  if (rc) return rc;
  return launch_linear_f32x(qan32, w_qb, q, n, q_rank, NQ, stream, "q_b_proj");
}

int mla_o_proj(const mla_dims* dims, int32_t hidden_size, const void* attn, const void* w_o, int64_t n, void* out,
               cudaStream_t stream) {
  int rc = check_dims(dims);
  if (rc) return rc;
  rc = check_proj_rows(n);
  if (rc) return rc;
  if (hidden_size < 1) return fail(MLA_ERR_INVALID_ARG, "hidden_size must be >= 1");
  if (!attn || !w_o || !out) return fail(MLA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (n == 0) return MLA_OK;
  return launch_linear(dims, attn, w_o, out, n, dims->num_heads * dims->v_head, hidden_size, stream, "o_proj");
}

int mla_selftest_wait_timeout(uint32_t limit_us, int32_t* gave_up, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return fail(MLA_ERR_INVALID_ARG, "limit_us must be in 1 .. 1000000");
  if (!gave_up) return fail(MLA_ERR_INVALID_ARG, "gave_up is NULL");
  prof_begin(stream, "selftest_wait_timeout");
  mla::tc::wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000ull, gave_up);
  prof_end(stream);
  return cuda_status(cudaGetLastError(), "self-test launch");
}

int mla_check_device_status(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_status(e, "stream synchronize");
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, mla::g_device_error, sizeof(v));
  if (e != cudaSuccess) return cuda_status(e, "read device error word");
  if (v) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(mla::g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_status(e, "clear device error word");
    if (v & mla::kDevErrTimeout) return fail(MLA_ERR_DEVICE_TIMEOUT, "a device-side wait timed out (0x%x)", v);
    if (v & mla::kDevErrRange)
      return fail(MLA_ERR_INVALID_ARG, "a q, key or value exceeded the fp16 range of the internal buffers (0x%x)", v);
    return fail(MLA_ERR_INVALID_ARG, "device-side input check failed (0x%x)", v);
  }
  return MLA_OK;
}

}  // extern "C"
