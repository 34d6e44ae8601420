// bd_masked_ce: the masked-token cross-entropy of training with the shifted
// label ("Fast-dLLM v2: Efficient Block-Diffusion LLM", key design 2, the
// L_block equation): in each training sequence, every position i >= 1 that
// is [MASK] in the noisy stream contributes
//
//     -log softmax(W h_{i-1})[x_0^i] = max_v l_v + log sum_v exp(l_v - max) - l_y,
//
// l = W h_{i-1}, y = x_0^i; position 0 has no previous row and contributes
// nothing.  The logits never reach memory: the LM head's (max, sum exp)
// fold is the one of bd_confidence_select.
//
// Launches (each after the first chained by programmatic dependent launch):
//   1. ce_gather   packs row i-1 of every scored position into [M][H], with
//                  the position and its target per packed row; writes NaN
//                  to the loss of every unscored position;
//   2. LM head     (max, sum exp) per packed row, vocab-split partials
//                  (tcgen05 for bf16: rows as the M operand from 2048 rows
//                  up, W as the M operand below; CUDA cores for fp32);
//   3. ce_merge    per row: merge the partials, the target logit as a dot
//                  product of W[y] and the row, the loss;
//   4. ce_sum      one CTA adds the losses in row order (a deterministic
//                  sum) and writes the count.
#include "bd_common.cuh"

namespace bd {
namespace {

// 8 consecutive elements as fp32 (16-byte loads; rows are 16-byte aligned).
__device__ __forceinline__ void load8f(const bf16* p, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}
__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

// grid (n_words), 1024 threads: word x covers positions 32 x .. 32 x + 31 of
// the flattened [n_seqs * seq_len] stream; warp i handles position 32 x + i.
template <typename T>
__global__ void __launch_bounds__(1024) ce_gather_kernel(
    const T* __restrict__ h, const int32_t* __restrict__ targets,
    const uint32_t* __restrict__ masked, int n_words, int seq_words, int H, T* __restrict__ rows,
    int32_t* __restrict__ rowpos, int32_t* __restrict__ tgt, int32_t* __restrict__ count,
    float* __restrict__ loss_out, int rows_alloc) {
  __shared__ int red[32];
  griddep_wait();  // first kernel of the call: the caller's inputs are complete after this
  griddep_launch_dependents();
  const int x = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int acc = 0;
  for (int y = threadIdx.x; y < x; y += blockDim.x) acc += __popc(ce_scored_bits(masked[y], y, seq_words));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  int off = 0;
#pragma unroll
  for (int w = 0; w < 32; ++w) off += red[w];
  const uint32_t bits = ce_scored_bits(masked[x], x, seq_words);
  const int i = warp;
  const size_t p = static_cast<size_t>(x) * kBlock + i;  // position in the flat stream
  const bool scored = (bits >> i) & 1u;
  if (!scored) {
    if (lane == 0 && loss_out) loss_out[p] = __int_as_float(0x7fc00000);
  } else {
    const int r = off + __popc(bits & ((1u << i) - 1u));
    if (lane == 0) {
      rowpos[r] = static_cast<int32_t>(p);
      tgt[r] = targets[p];
    }
    const uint4* s4 = reinterpret_cast<const uint4*>(h + (p - 1) * H);  // row i-1, same sequence
    uint4* d4 = reinterpret_cast<uint4*>(rows + static_cast<size_t>(r) * H);
    const int nvec = H * static_cast<int>(sizeof(T)) / 16;
    for (int v = lane; v < nvec; v += 32) d4[v] = s4[v];
  }
  if (x == n_words - 1) {
    const int total = off + __popc(bits);
    if (threadIdx.x == 0) {
      count[0] = total;
      count[1] = 0;  // status word of the tensor-core LM head
    }
    const int pad_end = min(rows_alloc, (total + 15) / 16 * 16);
    const int nvec = (pad_end - total) * H * static_cast<int>(sizeof(T)) / 16;
    uint4* d4 = reinterpret_cast<uint4*>(rows + static_cast<size_t>(total) * H);
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) d4[v] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// grid (rows_alloc / 8), 256 threads: warp per packed row.  parts = the
// row's partials (n_split, or n_split / G for the tensor-core LM head's G
// row groups of <= 256).
template <typename T>
__global__ void __launch_bounds__(256) ce_merge_kernel(
    const T* __restrict__ rows, const T* __restrict__ w, const int32_t* __restrict__ rowpos,
    const int32_t* __restrict__ tgt, const int32_t* __restrict__ count, int n_split, int grouped,
    const float* __restrict__ pm, const float* __restrict__ ps, int H, int V,
    float* __restrict__ loss_row, float* __restrict__ loss_out) {
  griddep_wait();  // the LM head's partials
  griddep_launch_dependents();
  const int M = count[0];
  const int r = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (r >= M) return;
  const int parts = grouped ? n_split / ((M + 255) / 256) : n_split;
  Stat st = stat_empty();
  const size_t base = static_cast<size_t>(r) * n_split;
  for (int k = lane; k < parts; k += 32) st = stat_combine(st, Stat{pm[base + k], ps[base + k], 0});
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const Stat other{__shfl_xor_sync(0xffffffffu, st.m, o), __shfl_xor_sync(0xffffffffu, st.s, o), 0};
    st = stat_combine(st, other);
  }
  const int y = tgt[r];
  if (lane == 0) BD_CHECK(y >= 0 && y < V, kCheckTargetId, y);
  float dot = 0.f;
  if (y >= 0 && y < V) {
    const T* wr = w + static_cast<size_t>(y) * H;
    const T* hr = rows + static_cast<size_t>(r) * H;
    for (int k = lane * 8; k < H; k += 256) {
      float a[8], b[8];
      load8f(wr + k, a);
      load8f(hr + k, b);
#pragma unroll
      for (int e = 0; e < 8; ++e) dot = fmaf(a[e], b[e], dot);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if (lane == 0) {
    const bool ok = count[1] == 0 && y >= 0 && y < V && st.s > 0.f;
    const float loss = ok ? st.m + logf(st.s) - dot : __int_as_float(0x7fc00000);
    loss_row[r] = loss;
    if (loss_out) loss_out[rowpos[r]] = loss;
  }
}

// one CTA of 1024 threads: the sum of the M row losses in row order.
__global__ void __launch_bounds__(1024) ce_sum_kernel(const float* __restrict__ loss_row,
                                                      const int32_t* __restrict__ count,
                                                      float* __restrict__ loss_sum,
                                                      int32_t* __restrict__ n_scored) {
  __shared__ float red[32];
  griddep_wait();  // the per-row losses
  griddep_launch_dependents();
  const int M = count[0];
  float acc = 0.f;
  for (int r = threadIdx.x; r < M; r += blockDim.x) acc += loss_row[r];
  acc = warp_sum(acc);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = red[threadIdx.x];
    v = warp_sum(v);
    if (threadIdx.x == 0) {
      *loss_sum = v;
      if (n_scored) *n_scored = M;
    }
  }
}

// bf16 LM head: rows as the MMA's M operand from 2048 packed rows up (W is
// then streamed about once); below that W as the M operand, the rows
// re-read per vocab tile.
constexpr int kCeRowsMin = 2048;
bool ce_use_rows(int dtype, int rows_alloc) {
  return dtype == BD_BF16 && rows_alloc >= kCeRowsMin;
}
bool ce_use_tc(int dtype, int rows_alloc) {
  return dtype == BD_BF16 && (rows_alloc + 255) / 256 <= lmhead_tc_grid();
}

}  // namespace

CePlan plan_masked_ce(int dtype, int n_seqs, int seq_len, int hidden, int vocab) {
  CePlan p{};
  const size_t positions = static_cast<size_t>(n_seqs) * seq_len;
  p.rows_alloc = static_cast<int>(align_up(positions, 256));
  p.rows = ce_use_rows(dtype, p.rows_alloc);
  p.tc = !p.rows && ce_use_tc(dtype, p.rows_alloc);
  p.n_split = p.rows ? 2 * lmhead_rows_ranges(vocab)
                     : (p.tc ? lmhead_tc_grid() : lmhead_simt_splits(vocab, p.rows_alloc));
  const size_t es = dtype == BD_BF16 ? 2 : 4;
  const size_t ra = static_cast<size_t>(p.rows_alloc);
  size_t off = 0;
  p.off_count = off;  // [0] = M, [1] = status word of the tensor-core LM head
  off = align_up(off + 16, 256);
  p.off_rows = off;
  off = align_up(off + ra * hidden * es, 256);
  p.off_rowpos = off;
  off = align_up(off + ra * 4, 256);
  p.off_tgt = off;
  off = align_up(off + ra * 4, 256);
  const size_t part = static_cast<size_t>(p.n_split) * ra * 4;
  p.off_pm = off;
  off = align_up(off + part, 256);
  p.off_ps = off;
  off = align_up(off + part, 256);
  p.off_pa = off;
  off = align_up(off + part, 256);
  p.off_loss = off;
  off = align_up(off + ra * 4, 256);
  p.total = off;
  return p;
}

template <typename T>
static cudaError_t launch_ce_t(int n_seqs, int seq_len, int hidden, int vocab, const CePlan& p,
                               const void* h, const void* w, const int32_t* targets,
                               const uint32_t* masked, float* loss_out, float* loss_sum,
                               int32_t* n_scored, void* ws, cudaStream_t st) {
  char* base = static_cast<char*>(ws);
  int32_t* count = reinterpret_cast<int32_t*>(base + p.off_count);
  T* rows = reinterpret_cast<T*>(base + p.off_rows);
  int32_t* rowpos = reinterpret_cast<int32_t*>(base + p.off_rowpos);
  int32_t* tgt = reinterpret_cast<int32_t*>(base + p.off_tgt);
  float* pm = reinterpret_cast<float*>(base + p.off_pm);
  float* ps = reinterpret_cast<float*>(base + p.off_ps);
  int32_t* pa = reinterpret_cast<int32_t*>(base + p.off_pa);
  float* loss_row = reinterpret_cast<float*>(base + p.off_loss);
  const int seq_words = seq_len / kBlock;
  const int n_words = n_seqs * seq_words;
  cudaError_t e = launch_pdl(ce_gather_kernel<T>, dim3(n_words), dim3(1024), 0, st,
                             static_cast<const T*>(h), targets, masked, n_words, seq_words, hidden,
                             rows, rowpos, tgt, count, loss_out, p.rows_alloc);
  if (e != cudaSuccess) return e;
  count_launches(1);
  if (p.rows) {
    e = launch_lmhead_rows(rows, w, masked, n_words, seq_words, hidden, vocab, p.rows_alloc,
                           p.n_split / 2, pm, ps, count + 1, st);
  } else if (p.tc) {
    e = launch_lmhead_tc(rows, w, masked, n_words, kBlock, 0, hidden, vocab, p.rows_alloc,
                         p.n_split, pm, ps, pa, count + 1, st, seq_words);
  } else {
    e = launch_lmhead_simt(sizeof(T) == 2 ? BD_BF16 : BD_F32, rows, w, count, hidden, vocab,
                           p.n_split, p.rows_alloc, pm, ps, pa, st);
  }
  if (e != cudaSuccess) return e;
  e = launch_pdl(ce_merge_kernel<T>, dim3(p.rows_alloc / 8), dim3(256), 0, st,
                 static_cast<const T*>(rows), static_cast<const T*>(w),
                 static_cast<const int32_t*>(rowpos), static_cast<const int32_t*>(tgt),
                 static_cast<const int32_t*>(count), p.n_split, p.tc ? 1 : 0,
                 static_cast<const float*>(pm), static_cast<const float*>(ps), hidden, vocab,
                 loss_row, loss_out);
  if (e != cudaSuccess) return e;
  count_launches(1);
  e = launch_pdl(ce_sum_kernel, dim3(1), dim3(1024), 0, st, static_cast<const float*>(loss_row),
                 static_cast<const int32_t*>(count), loss_sum, n_scored);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_masked_ce(int dtype, int n_seqs, int seq_len, int hidden, int vocab,
                             const CePlan& p, const void* h, const void* w, const int32_t* targets,
                             const uint32_t* masked, float* loss_out, float* loss_sum,
                             int32_t* n_scored, void* ws, cudaStream_t st) {
  if (dtype == BD_BF16)
    return launch_ce_t<bf16>(n_seqs, seq_len, hidden, vocab, p, h, w, targets, masked, loss_out,
                             loss_sum, n_scored, ws, st);
  return launch_ce_t<float>(n_seqs, seq_len, hidden, vocab, p, h, w, targets, masked, loss_out,
                            loss_sum, n_scored, ws, st);
}

}  // namespace bd

#ifdef BD_DEVICE_CHECKS
namespace bd {
cudaError_t check_word_ce(int* host2, bool reset) { return read_check_word(host2, reset); }
}  // namespace bd
#endif
