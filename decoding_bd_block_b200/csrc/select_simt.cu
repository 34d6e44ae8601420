// bd_confidence_select: token shift -> LM head -> (max, sum, argmax) per row
// -> confidence-aware unmask ("Fast-dLLM v2: Efficient Block-Diffusion LLM",
// key designs 2-4; Fast-dLLM v1 article, confidence-aware parallel decoding).
//
// Launches:
//   1. gather_rows     packs, per masked position i, hidden row i-1 (h_prev
//                      for i = 0) into a dense [M][H] matrix (one warp per
//                      position, 16-byte copies); records each position's
//                      row and M;
//   2. LM-head stats   vocab-split: each CTA folds its vocab range into a
//                      running (max, sum exp, argmax) per row; logits stay on
//                      chip (tcgen05 in select_tc.cu for bf16; the CUDA-core
//                      tile below for fp32);
//   3. merge_select    one warp per position merges that row's partials,
//                      turns them into p_max and the token; warp 0 then
//                      applies the unmask rule of the sequence.
// Partials are stored [row][part] so a row's partials are contiguous.
#include "bd_common.cuh"

namespace bd {

// grid (batch), 1024 threads: warp i copies the row of position i.
template <typename T>
__global__ void __launch_bounds__(1024) gather_rows_kernel(
    const T* __restrict__ h, const T* __restrict__ h_prev, const uint32_t* __restrict__ masked,
    int B, int H, T* __restrict__ rows, int32_t* __restrict__ posrow,
    int32_t* __restrict__ count, int rows_alloc, int S, int active) {
  __shared__ int red[32];
  griddep_wait();  // first kernel of the call: the caller's inputs are complete after this
  griddep_launch_dependents();
  const int s = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int acc = 0;
  for (int x = threadIdx.x; x < s; x += blockDim.x) acc += __popc(scored_bits(masked[x], S, active));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  int off = 0;
#pragma unroll
  for (int w = 0; w < 32; ++w) off += red[w];
  const uint32_t bits = scored_bits(masked[s], S, active);
  const int i = warp;
  const bool is_m = (bits >> i) & 1u;
  const int r = is_m ? off + __popc(bits & ((1u << i) - 1u)) : -1;
  if (lane == 0) posrow[s * kBlock + i] = r;
  if (is_m) {
    const T* src = (i == 0) ? h_prev + static_cast<size_t>(s) * H
                            : h + (static_cast<size_t>(s) * kBlock + i - 1) * H;
    T* dst = rows + static_cast<size_t>(r) * H;
    const int nvec = H * static_cast<int>(sizeof(T)) / 16;  // H * sizeof(T) % 16 == 0
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    // eight 16-byte loads in flight per lane before their stores
    for (int x0 = lane; x0 < nvec; x0 += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (x0 + 32 * u < nvec) v[u] = s4[x0 + 32 * u];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (x0 + 32 * u < nvec) d4[x0 + 32 * u] = v[u];
    }
  }
  if (s == B - 1) {
    const int total = off + __popc(bits);
    if (threadIdx.x == 0) {
      count[0] = total;
      count[1] = 0;  // status word of the LM-head kernel
    }
    const int pad_end = min(rows_alloc, (total + 15) / 16 * 16);
    const int nvec = (pad_end - total) * H * static_cast<int>(sizeof(T)) / 16;
    uint4* d4 = reinterpret_cast<uint4*>(rows + static_cast<size_t>(total) * H);
    for (int x = threadIdx.x; x < nvec; x += blockDim.x) d4[x] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// grid (n_split, rows_alloc / 32), 256 threads.  Tile: 64 vocab x 32 rows,
// K-steps of 32; CTA x strides over vocab tiles x, x + n_split, ...
template <typename T>
__global__ void __launch_bounds__(256) lmhead_simt_kernel(
    const T* __restrict__ rows, const T* __restrict__ w, const int32_t* __restrict__ count,
    int H, int V, int n_split, float* __restrict__ pm, float* __restrict__ ps,
    int32_t* __restrict__ pa) {
  __shared__ float Ws[32][68];
  __shared__ float Rs[32][36];
  __shared__ float Ls[32][65];
  const int M = *count;
  const int r0 = blockIdx.y * 32;
  if (r0 >= M) return;
  const int tid = threadIdx.x;
  const int tv = tid % 16, tr = tid / 16;
  float run_m = -INFINITY, run_s = 0.f;
  int run_a = 0x7fffffff;
  for (int vt = blockIdx.x; vt * 64 < V; vt += n_split) {
    const int v0 = vt * 64;
    float acc[2][4] = {};
    for (int k0 = 0; k0 < H; k0 += 32) {
      __syncthreads();
      for (int i = tid; i < 64 * 32; i += 256) {
        const int vv = i / 32, kk = i % 32;
        const int vg = v0 + vv, kg = k0 + kk;
        Ws[kk][vv] = (vg < V && kg < H) ? to_f32(w[static_cast<size_t>(vg) * H + kg]) : 0.f;
      }
      for (int i = tid; i < 32 * 32; i += 256) {
        const int rr = i / 32, kk = i % 32;
        const int rg = r0 + rr, kg = k0 + kk;
        Rs[kk][rr] = (rg < M && kg < H) ? to_f32(rows[static_cast<size_t>(rg) * H + kg]) : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < 32; ++kk) {
        float wv[4], rv[2];
#pragma unroll
        for (int b = 0; b < 4; ++b) wv[b] = Ws[kk][tv * 4 + b];
#pragma unroll
        for (int a = 0; a < 2; ++a) rv[a] = Rs[kk][tr * 2 + a];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(rv[a], wv[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) Ls[tr * 2 + a][tv * 4 + b] = acc[a][b];
    __syncthreads();
    if (tid < 32) {
      for (int vv = 0; vv < 64 && v0 + vv < V; ++vv) {
        const float x = Ls[tid][vv];
        if (x > run_m) {
          run_s = run_s * expf(run_m - x) + 1.f;
          run_m = x;
          run_a = v0 + vv;
        } else {
          run_s += expf(x - run_m);
        }
      }
    }
  }
  if (tid < 32 && r0 + tid < M) {
    const size_t idx = static_cast<size_t>(r0 + tid) * n_split + blockIdx.x;
    pm[idx] = run_m;
    ps[idx] = run_s;
    pa[idx] = run_a;
  }
}

// grid (batch), 1024 threads: warp i merges the partials of position i.
// With grouped partials (tensor-core LM head) each row has n_split / G
// parts, G = ceil(M / 256) row groups.  A nonzero status word (a bounded
// wait gave up) turns the outputs into "no decision": nothing is unmasked,
// p_max is NaN and the token -2.
__global__ void __launch_bounds__(1024) merge_select_kernel(
    const int32_t* __restrict__ posrow, const int32_t* __restrict__ count,
    const uint32_t* __restrict__ masked, int n_split, int grouped, const float* __restrict__ pm,
    const float* __restrict__ ps, const int32_t* __restrict__ pa, float tau, int S,
    int32_t* __restrict__ tokens, uint32_t* __restrict__ unmask, float* __restrict__ pmax_out,
    int32_t* __restrict__ argmax_out, int active) {
  __shared__ float sp[kBlock];
  __shared__ int stok[kBlock];
  griddep_wait();  // the LM head's partials
  griddep_launch_dependents();
  const int s = blockIdx.x;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t bits = scored_bits(masked[s], S, active);
  if (count[1] != 0) {
    if (warp == 0) no_decision_sequence(s, unmask, pmax_out, argmax_out);
    return;
  }
  const int parts = grouped ? n_split / ((count[0] + 255) / 256) : n_split;
  {
    // Two passes over the row's partials, all of a lane's loads in flight:
    // the largest max, then sum exp and the lowest argmax attaining it.
    constexpr int kPer = 8;  // partials per lane kept in registers (parts <= 256)
    const int i = warp;
    float s_sum = 0.f;
    int a_min = 0x7fffffff;
    float M = -INFINITY;
    if ((bits >> i) & 1u) {
      int prow = posrow[s * kBlock + i];
      if (lane == 0) BD_CHECK(prow >= 0 && prow < count[0], kCheckRowIndex, prow);
      prow = (prow >= 0 && prow < count[0]) ? prow : 0;  // written by the gather kernel
      const size_t base = static_cast<size_t>(prow) * n_split;
      float m[kPer], sv[kPer];
      int av[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int k = lane + 32 * u;
        const bool in = k < parts;
        m[u] = in ? pm[base + k] : -INFINITY;
        sv[u] = in ? ps[base + k] : 0.f;
        av[u] = in ? pa[base + k] : 0x7fffffff;
      }
      for (int k = lane + 32 * kPer; k < parts; k += 32) {  // more than 256 partials
        const Stat x = stat_combine(Stat{m[0], sv[0], av[0]}, Stat{pm[base + k], ps[base + k], pa[base + k]});
        m[0] = x.m;
        sv[0] = x.s;
        av[0] = x.a;
      }
      float lm = m[0];
#pragma unroll
      for (int u = 1; u < kPer; ++u) lm = fmaxf(lm, m[u]);
      M = warp_max(lm);
      if (M != -INFINITY) {
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          if (m[u] != -INFINITY) s_sum += sv[u] * exp2f((m[u] - M) * kLog2e);
          if (m[u] == M) a_min = min(a_min, av[u]);
        }
      }
      s_sum = warp_sum(s_sum);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a_min = min(a_min, __shfl_xor_sync(0xffffffffu, a_min, o));
    }
    if (lane == 0) {
      sp[i] = s_sum > 0.f ? 1.f / s_sum : 0.f;
      stok[i] = a_min;
    }
  }
  __syncthreads();
  if (warp != 0) return;
  select_sequence(s, bits, sp[lane], stok[lane], tau, S, tokens, unmask, pmax_out, argmax_out);
}

// -------------------------------------------------------------- host side
cudaError_t launch_lmhead_simt(int dtype, const void* rows, const void* w, const int32_t* count,
                               int H, int V, int n_split, int rows_alloc, float* pm, float* ps,
                               int32_t* pa, cudaStream_t st) {
  if (dtype == BD_BF16)
    lmhead_simt_kernel<bf16><<<dim3(n_split, rows_alloc / 32), 256, 0, st>>>(
        static_cast<const bf16*>(rows), static_cast<const bf16*>(w), count, H, V, n_split, pm, ps,
        pa);
  else
    lmhead_simt_kernel<float><<<dim3(n_split, rows_alloc / 32), 256, 0, st>>>(
        static_cast<const float*>(rows), static_cast<const float*>(w), count, H, V, n_split, pm,
        ps, pa);
  count_launches(1);
  return cudaGetLastError();
}

// vocab splits of the CUDA-core LM head: about four CTAs per SM over the
// (split, 32-row tile) grid
int lmhead_simt_splits(int vocab, int rows_alloc) {
  const int vtiles = (vocab + 63) / 64;
  const int rtiles = rows_alloc / 32;
  int ns = (4 * 148 + rtiles - 1) / rtiles;
  if (ns > vtiles) ns = vtiles;
  if (ns < 1) ns = 1;
  return ns;
}

// The tensor-core LM head takes bf16 whenever every row group of <= 256 rows
// still gets at least one vocab range of its own.
static bool use_tc(int dtype, int batch) {
  return dtype == BD_BF16 && (batch * kBlock + 255) / 256 <= lmhead_tc_grid();
}

SelectPlan plan_confidence_select(int dtype, int batch, int hidden, int vocab) {
  SelectPlan p{};
  p.rows_alloc = static_cast<int>(align_up(static_cast<size_t>(batch) * kBlock, 256));
  p.fused = select_fused_supported(dtype, batch, hidden);
  p.tc = use_tc(dtype, batch);
  if (p.fused) {
    p.rows_alloc = kBlock;  // partials per position of the one sequence
    p.n_split = select_fused_part_stride();
  } else if (p.tc) {
    p.n_split = lmhead_tc_grid();
  } else {
    p.n_split = lmhead_simt_splits(vocab, p.rows_alloc);
  }
  const size_t es = dtype == BD_BF16 ? 2 : 4;
  size_t off = 0;
  // Header, zero between calls: [0] = M, [1] = status word of the
  // tensor-core kernels, [2] = CTA arrivals and [3] = vocab-tile counter of
  // the single-kernel path.
  p.off_count = off;
  off = align_up(off + 16, 256);
  p.off_rows = off;
  if (!p.fused) off = align_up(off + static_cast<size_t>(p.rows_alloc) * hidden * es, 256);
  p.off_posrow = off;
  if (!p.fused) off = align_up(off + static_cast<size_t>(batch) * kBlock * 4, 256);
  const size_t part = static_cast<size_t>(p.n_split) * p.rows_alloc * 4;
  p.off_pm = off;
  off = align_up(off + part, 256);
  p.off_ps = off;
  off = align_up(off + part, 256);
  p.off_pa = off;
  off = align_up(off + part, 256);
  p.total = off;
  return p;
}

template <typename T>
static cudaError_t launch_select_t(int batch, int hidden, int vocab, const SelectPlan& p,
                                   const void* h, const void* h_prev, const void* w,
                                   const uint32_t* masked, float tau, int S, int32_t* tokens,
                                   uint32_t* unmask, float* pmax_out, int32_t* argmax_out,
                                   void* ws, cudaStream_t st, int active) {
  char* base = static_cast<char*>(ws);
  T* rows = reinterpret_cast<T*>(base + p.off_rows);
  int32_t* posrow = reinterpret_cast<int32_t*>(base + p.off_posrow);
  int32_t* count = reinterpret_cast<int32_t*>(base + p.off_count);
  float* pm = reinterpret_cast<float*>(base + p.off_pm);
  float* ps = reinterpret_cast<float*>(base + p.off_ps);
  int32_t* pa = reinterpret_cast<int32_t*>(base + p.off_pa);
  if (p.fused)
    return launch_select_fused(hidden, vocab, h, h_prev, w, masked, tau, S, tokens, unmask,
                               pmax_out, argmax_out, pm, ps, pa, count, active, st);
  cudaError_t e = launch_pdl(gather_rows_kernel<T>, dim3(batch), dim3(1024), 0, st,
                             static_cast<const T*>(h), static_cast<const T*>(h_prev), masked,
                             batch, hidden, rows, posrow, count, p.rows_alloc, S, active);
  if (e != cudaSuccess) return e;
  count_launches(1);
  if (p.tc) {
    e = launch_lmhead_tc(rows, w, masked, batch, S, active, hidden, vocab, p.rows_alloc,
                         p.n_split, pm, ps, pa, count + 1, st);
    if (e != cudaSuccess) return e;
  } else {
    lmhead_simt_kernel<T><<<dim3(p.n_split, p.rows_alloc / 32), 256, 0, st>>>(
        rows, static_cast<const T*>(w), count, hidden, vocab, p.n_split, pm, ps, pa);
    count_launches(1);
  }
  e = launch_pdl(merge_select_kernel, dim3(batch), dim3(1024), 0, st, posrow,
                 static_cast<const int32_t*>(count), masked, p.n_split, p.tc ? 1 : 0,
                 static_cast<const float*>(pm), static_cast<const float*>(ps),
                 static_cast<const int32_t*>(pa), tau, S, tokens, unmask, pmax_out, argmax_out,
                 active);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_confidence_select(int dtype, int batch, int hidden, int vocab,
                                     const SelectPlan& p, const void* h, const void* h_prev,
                                     const void* w, const uint32_t* masked, float tau,
                                     int sub_block, int32_t* tokens, uint32_t* unmask,
                                     float* pmax_out, int32_t* argmax_out, void* ws,
                                     cudaStream_t st, int active) {
  if (dtype == BD_BF16)
    return launch_select_t<bf16>(batch, hidden, vocab, p, h, h_prev, w, masked, tau, sub_block,
                                 tokens, unmask, pmax_out, argmax_out, ws, st, active);
  return launch_select_t<float>(batch, hidden, vocab, p, h, h_prev, w, masked, tau, sub_block,
                                tokens, unmask, pmax_out, argmax_out, ws, st, active);
}

}  // namespace bd

#ifdef BD_DEVICE_CHECKS
namespace bd {
cudaError_t check_word_select(int* host2, bool reset) { return read_check_word(host2, reset); }
}  // namespace bd
#endif
