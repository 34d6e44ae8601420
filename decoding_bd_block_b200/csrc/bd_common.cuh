// Shared device helpers of libbd (element access, RoPE angles, fast exp2,
// warp reductions) and the internal launcher interface used by bd_api.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/bd.h"

namespace bd {

using bf16 = __nv_bfloat16;

constexpr int kBlock = BD_BLOCK;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- elements
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// 2^x on the MUFU unit (hardware approximation, relative error ~2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, for spreading exponentials over MUFU and FMA units.
// Round-to-nearest split x = j + f, |f| <= 1/2 (adding 1.5 * 2^23 leaves
// round(x) in the low mantissa bits); 2^f from a degree-4 polynomial fitted
// to 2^f on [-1/2, 1/2] by weighted least squares on Chebyshev nodes (max
// relative error 2.6e-6 in exact arithmetic, 2.7e-6 once the Horner steps
// round in fp32: measured against 2^x in double precision over [-126, 0]);
// 2^j is added to the exponent field.  Inputs below -126 return 2^-126.
__device__ __forceinline__ float poly_exp2(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const int j = __float_as_int(t) - 0x4B400000;
  const float f = x - (t - 12582912.f);
  float p = fmaf(0.009570101434f, f, 0.05591786028f);
  p = fmaf(p, f, 0.2402474484f);
  p = fmaf(p, f, 0.6931218147f);
  p = fmaf(p, f, 0.9999992614f);
  return __int_as_float(__float_as_int(p) + j * (1 << 23));
}

// Paired fp32 arithmetic (two lanes of a 64-bit register pair per
// instruction, sm_100): d = a * b + c and d = a + b, each lane rounded as the
// scalar instruction would be.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// poly_exp2 on a pair, the polynomial in paired arithmetic.
__device__ __forceinline__ float2 poly_exp2x2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = fadd2(x, make_float2(12582912.f, 12582912.f));
  const int jx = __float_as_int(t.x) - 0x4B400000, jy = __float_as_int(t.y) - 0x4B400000;
  const float2 u = fadd2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = ffma2(u, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(make_float2(0.009570101434f, 0.009570101434f), f,
                   make_float2(0.05591786028f, 0.05591786028f));
  p = ffma2(p, f, make_float2(0.2402474484f, 0.2402474484f));
  p = ffma2(p, f, make_float2(0.6931218147f, 0.6931218147f));
  p = ffma2(p, f, make_float2(0.9999992614f, 0.9999992614f));
  return make_float2(__int_as_float(__float_as_int(p.x) + jx * (1 << 23)),
                     __int_as_float(__float_as_int(p.y) + jy * (1 << 23)));
}

// The same, also raising jmax to the larger integer part round(x) of the
// pair (the polynomial's result is 2^x only while that is below 128).
__device__ __forceinline__ float2 poly_exp2x2(float2 x, int& jmax) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = fadd2(x, make_float2(12582912.f, 12582912.f));
  const int jx = __float_as_int(t.x) - 0x4B400000, jy = __float_as_int(t.y) - 0x4B400000;
  jmax = __vimax3_s32(jmax, jx, jy);
  const float2 u = fadd2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = ffma2(u, make_float2(-1.f, -1.f), x);
  float2 p = ffma2(make_float2(0.009570101434f, 0.009570101434f), f,
                   make_float2(0.05591786028f, 0.05591786028f));
  p = ffma2(p, f, make_float2(0.2402474484f, 0.2402474484f));
  p = ffma2(p, f, make_float2(0.6931218147f, 0.6931218147f));
  p = ffma2(p, f, make_float2(0.9999992614f, 0.9999992614f));
  return make_float2(__int_as_float(__float_as_int(p.x) + jx * (1 << 23)),
                     __int_as_float(__float_as_int(p.y) + jy * (1 << 23)));
}

// ------------------------------------------- programmatic dependent launch
// A kernel launched with launch_pdl() may start while the previous kernel of
// the stream is still running: it must call griddep_wait() before it reads
// anything that kernel writes (and before it writes anything that kernel
// reads).  griddep_launch_dependents() lets the next PDL kernel start early.
// Both are no-ops for a kernel launched the ordinary way.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// --------------------------------------------------------------- warp ops
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ------------------------------------------------------------------ RoPE
// cos/sin of pos * theta^(-2j/d), evaluated in double precision so that the
// angle stays exact to ~1e-12 rad at positions in the tens of thousands.
__device__ __forceinline__ void rope_cos_sin(long long pos, double inv_freq, float* c, float* s) {
  double sd, cd;
  sincos(static_cast<double>(pos) * inv_freq, &sd, &cd);
  *c = static_cast<float>(cd);
  *s = static_cast<float>(sd);
}

__device__ __forceinline__ double rope_inv_freq(int j, int d, double theta) {
  return pow(theta, -2.0 * static_cast<double>(j) / static_cast<double>(d));
}

// theta^(-2j/d) for j < d/2, computed on the host in double precision and
// passed by value, so that a kernel needs no pow.
struct RopeFreq {
  double inv[64];
};
void rope_freq_table(int d, double theta, RopeFreq* f);

// ------------------------------------------------- (max, sum, argmax) triple
// Running softmax statistics of a set of logits: m = max, s = sum exp(l - m),
// a = lowest index attaining m.  combine() is associative and commutative.
struct Stat {
  float m;
  float s;
  int a;
};
__device__ __forceinline__ Stat stat_empty() { return Stat{-INFINITY, 0.f, 0x7fffffff}; }
__device__ __forceinline__ Stat stat_combine(Stat x, Stat y) {
  if (y.m == -INFINITY) return x;
  if (x.m == -INFINITY) return y;
  Stat r;
  r.m = fmaxf(x.m, y.m);
  r.s = x.s * expf(x.m - r.m) + y.s * expf(y.m - r.m);
  if (x.m == y.m) r.a = min(x.a, y.a);
  else r.a = (x.m > y.m) ? x.a : y.a;
  return r;
}

// ------------------------------------------ confidence-aware unmask rule
// One sequence on one warp: lane i holds position i's mask bit (bit i of
// `bits`), its p_max and its argmax token.  Candidates are the masked
// positions of the lowest sub-block of S positions that still has one; every
// candidate with p_max > tau is unmasked, or the most confident candidate
// (lowest position on ties) when none is ("Fast-dLLM v2: Efficient
// Block-Diffusion LLM", key design 4; Fast-dLLM v1 article, confidence-aware
// parallel decoding).  Writes the chosen tokens, the unmask bits and, when
// given, p_max / argmax (NaN / -1 at unmasked positions).
__device__ __forceinline__ void select_sequence(int s, uint32_t bits, float p, int tok, float tau,
                                                int S, int32_t* tokens, uint32_t* unmask,
                                                float* pmax_out, int32_t* argmax_out) {
  const int i = threadIdx.x % 32;
  const bool is_m = (bits >> i) & 1u;
  p = is_m ? p : 0.f;
  tok = is_m ? tok : -1;
  const int first = bits ? __ffs(static_cast<int>(bits)) - 1 : 0;
  const int k0 = (first / S) * S;
  const bool cand = is_m && i >= k0 && i < k0 + S;
  const uint32_t above = __ballot_sync(0xffffffffu, cand && p > tau);
  uint32_t U = above;
  if (!above) {
    float bp = cand ? p : -1.f;
    int bi = cand ? i : 32;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float op = __shfl_xor_sync(0xffffffffu, bp, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (op > bp || (op == bp && oi < bi)) {
        bp = op;
        bi = oi;
      }
    }
    U = (bi < 32) ? (1u << bi) : 0u;
  }
  if ((U >> i) & 1u) tokens[s * kBlock + i] = tok;
  if (i == 0) unmask[s] = U;
  if (pmax_out) pmax_out[s * kBlock + i] = is_m ? p : __int_as_float(0x7fc00000);
  if (argmax_out) argmax_out[s * kBlock + i] = is_m ? tok : -1;
}

// The positions one step scores: every masked position, or -- active-only
// scoring -- the masked positions of the lowest sub-block of S positions
// that still has one, the only candidates the unmask rule can pick.
__device__ __forceinline__ uint32_t scored_bits(uint32_t bits, int S, int active) {
  if (!active || !bits) return bits;
  const int k0 = ((__ffs(static_cast<int>(bits)) - 1) / S) * S;
  const uint32_t win = S >= 32 ? 0xffffffffu : ((1u << S) - 1u) << k0;
  return bits & win;
}

// Cross-entropy rows of a training batch: word x of the mask bits covers
// positions 32 (x mod seq_words) .. +31 of one sequence; position 0 of a
// sequence has no previous hidden row and is not scored.
__device__ __forceinline__ uint32_t ce_scored_bits(uint32_t bits, int x, int seq_words) {
  return x % seq_words == 0 ? bits & ~1u : bits;
}

// "No decision" for sequence s (a bounded wait gave up): nothing is
// unmasked, p_max is NaN and the token -2.  Lane i of one warp writes position i.
__device__ __forceinline__ void no_decision_sequence(int s, uint32_t* unmask, float* pmax_out,
                                                     int32_t* argmax_out) {
  const int i = threadIdx.x % 32;
  if (i == 0) unmask[s] = 0u;
  if (pmax_out) pmax_out[s * kBlock + i] = __int_as_float(0x7fc00000);
  if (argmax_out) argmax_out[s * kBlock + i] = -2;
}

// ------------------------------------------------------ device-side checks
// Built with -DBD_DEVICE_CHECKS (the library variant libbd_checks.so), kernels
// check the indices they read from device memory (page ids, packed-row
// indices, target ids) before using them.  A failed check is handled as in
// the normal build (the access is skipped: zeros are read, nothing is
// written) and is also recorded in a status word {code, detail}, the first
// failure winning; bd_device_check_status() reports and clears it.  No trap,
// no fault: the kernel runs to completion.  Without the flag the checks
// compile to nothing.
enum : int { kCheckNone = 0, kCheckPageId = 1, kCheckRowIndex = 2, kCheckTargetId = 3 };
#ifdef BD_DEVICE_CHECKS
// one word per translation unit (internal linkage; read by check_word_<unit>)
static __device__ int g_check_word[2];
__device__ __forceinline__ void check_fail(int code, int detail) {
  if (atomicCAS(&g_check_word[0], 0, code) == 0) g_check_word[1] = detail;
}
#define BD_CHECK(ok, code, detail)        \
  do {                                    \
    if (!(ok)) ::bd::check_fail(code, detail); \
  } while (0)
static inline cudaError_t read_check_word(int* host2, bool reset) {
  cudaError_t e = cudaMemcpyFromSymbol(host2, g_check_word, sizeof(g_check_word));
  if (e == cudaSuccess && reset) {
    const int zero[2] = {0, 0};
    e = cudaMemcpyToSymbol(g_check_word, zero, sizeof(zero));
  }
  return e;
}
#else
#define BD_CHECK(ok, code, detail) \
  do {                             \
  } while (0)
#endif
// The check words of the units that check (defined only with the flag).
cudaError_t check_word_commit(int* host2, bool reset);
cudaError_t check_word_attn_tc(int* host2, bool reset);
cudaError_t check_word_attn_simt(int* host2, bool reset);
cudaError_t check_word_select(int* host2, bool reset);
cudaError_t check_word_ce(int* host2, bool reset);

// Process-wide count of kernels enqueued by the library (bd_kernel_launches).
void count_launches(int n);
// Records a CUDA error for bd_last_cuda_error_string(); returns BD_ERR_CUDA
// (BD_OK for cudaSuccess).
int report_cuda_error(cudaError_t e);

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch `kern` so that it may begin before the stream's previous kernel has
// finished (programmatic stream serialisation); see griddep_wait().  Only
// the second and later kernels of one C-ABI call are launched this way, so
// work enqueued before the call has always completed when they start.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace bd

// ---------------------------------------------------------------------------
// Internal launchers (defined in the kernel files, called by bd_api.cu).
// Arguments are validated by the caller; each returns cudaGetLastError().
// ---------------------------------------------------------------------------
namespace bd {

struct CommitArgs {
  int n_seqs;
  int n_new_blocks;
  int seq_ids[256];
  int first_block[256];  // n_blocks_host[s] before the commit
};

cudaError_t launch_cache_commit(const bd_attn_shape& sh, const bd_kv_cache& c, const void* k,
                                const void* v, const CommitArgs& a, cudaStream_t st);

// Block attention plan: pages per split-KV chunk and the largest chunk count.
struct AttnPlan {
  bool tc;  // tcgen05 path (bf16, head_dim 128, G * 32 <= 256 query rows)
  int pages_per_chunk;
  int max_chunks;
  size_t off_q, off_blk, off_o, off_ml, off_status, total;
};
// Tensor-core block attention (attn_tc.cu).
bool attn_tc_supported(const bd_attn_shape& sh);
int attn_tc_max_chunk_pages();
cudaError_t launch_attn_tc(const bd_attn_shape& sh, const bd_kv_cache& c, int ppc, int max_chunks,
                           const void* ws_q, const void* ws_blk, float* part_o, float* part_ml,
                           void* out, int32_t* status, cudaStream_t st);
AttnPlan plan_block_attn(const bd_attn_shape& sh, const bd_kv_cache& c);
cudaError_t launch_block_attn(const bd_attn_shape& sh, const bd_kv_cache& c, const AttnPlan& p,
                              const void* q, const void* k, const void* v, void* out, void* ws,
                              cudaStream_t st);

// Tensor-core LM head (select_tc.cu): persistent grid size and launcher.
// The packed-row count is the popcount of masked[0 .. batch).
int lmhead_tc_grid();
// seq_words > 0: the rows are cross-entropy rows (ce_scored_bits of the
// batch words), S and active unused.
cudaError_t launch_lmhead_tc(const void* rows, const void* w, const uint32_t* masked, int batch,
                             int S, int active, int H, int V, int rows_alloc, int part_stride,
                             float* pm, float* ps, int32_t* pa, int32_t* status, cudaStream_t st,
                             int seq_words = 0);

struct SelectPlan {
  bool fused;        // one kernel, rows resident in shared memory (select_fused.cu)
  bool tc;           // LM head on tcgen05 (bf16)
  int n_split;       // vocab splits (partials per row)
  int rows_alloc;    // packed-row capacity (>= 32 * batch, padded)
  size_t off_rows, off_posrow, off_count, off_pm, off_ps, off_pa, total;
};
SelectPlan plan_confidence_select(int dtype, int batch, int hidden, int vocab);

// Single-kernel select (select_fused.cu): bf16, one sequence.  Partials are
// [32 positions][select_fused_part_stride()]; header points at the zeroed
// workspace header ([1] status, [2] arrivals, [3] tile counter), left zero.
bool select_fused_supported(int dtype, int batch, int hidden);
int select_fused_part_stride();
cudaError_t launch_select_fused(int hidden, int vocab, const void* h, const void* h_prev,
                                const void* w, const uint32_t* masked, float tau, int sub_block,
                                int32_t* tokens, uint32_t* unmask, float* pmax_out,
                                int32_t* argmax_out, float* pm, float* ps, int32_t* pa,
                                int32_t* header, int active, cudaStream_t st);
// active != 0: score only the active sub-block's masked positions (see
// scored_bits); the decisions are the same, p_max / argmax elsewhere NaN / -1.
cudaError_t launch_confidence_select(int dtype, int batch, int hidden, int vocab,
                                     const SelectPlan& p, const void* h, const void* h_prev,
                                     const void* w, const uint32_t* masked, float tau,
                                     int sub_block, int32_t* tokens, uint32_t* unmask,
                                     float* pmax_out, int32_t* argmax_out, void* ws,
                                     cudaStream_t st, int active = 0);

// Tensor-core mask attention (mask_attn_tc.cu): bf16, head_dim 128, L % 128 == 0.
bool mask_attn_tc_supported(const bd_attn_shape& sh, int L);
cudaError_t launch_mask_attn_tc(const bd_attn_shape& sh, const void* q, const void* k,
                                const void* v, void* out, int n_seqs, int L, int block,
                                int32_t* status, cudaStream_t st);

// CUDA-core LM head (select_simt.cu): partials [row][n_split] of the first
// count[0] rows; n_split from lmhead_simt_splits.
cudaError_t launch_lmhead_simt(int dtype, const void* rows, const void* w, const int32_t* count,
                               int H, int V, int n_split, int rows_alloc, float* pm, float* ps,
                               int32_t* pa, cudaStream_t st);
int lmhead_simt_splits(int vocab, int rows_alloc);

// Masked-token cross-entropy (masked_ce.cu).
struct CePlan {
  bool tc;    // LM head on tcgen05 with W as the M operand (few rows)
  bool rows;  // LM head on tcgen05 with the rows as the M operand (many rows)
  int n_split, rows_alloc;
  size_t off_count, off_rows, off_rowpos, off_tgt, off_pm, off_ps, off_pa, off_loss, total;
};
// Rows-as-M LM head of the cross-entropy (ce_lmhead.cu): (max, sum exp)
// partials [row][2 R] over R vocab ranges; bf16, rows_alloc a multiple of 256.
int lmhead_rows_ranges(int vocab);
cudaError_t launch_lmhead_rows(const void* rows, const void* w, const uint32_t* masked,
                               int n_words, int seq_words, int H, int V, int rows_alloc, int R,
                               float* pm, float* ps, int32_t* status, cudaStream_t st);
CePlan plan_masked_ce(int dtype, int n_seqs, int seq_len, int hidden, int vocab);
cudaError_t launch_masked_ce(int dtype, int n_seqs, int seq_len, int hidden, int vocab,
                             const CePlan& p, const void* h, const void* w, const int32_t* targets,
                             const uint32_t* masked, float* loss_out, float* loss_sum,
                             int32_t* n_scored, void* ws, cudaStream_t st);

cudaError_t launch_block_mask_attn(const bd_attn_shape& sh, const void* q, const void* k,
                                   const void* v, void* out, int n_seqs, int L, int block,
                                   cudaStream_t st);

}  // namespace bd
