// LM-head statistics on the 5th-generation tensor cores (bf16 in, fp32
// accumulate), for bd_confidence_select.
//
// Each packed row r (the hidden row that predicts one masked position) needs
// max_v l, sum_v exp(l - max) and argmax_v of l = row . W[v] over the whole
// vocabulary ("Fast-dLLM v2: Efficient Block-Diffusion LLM", key design 3:
// confidence of a masked token; Fast-dLLM v1 article, core technique 2).
// The logits never leave the chip:
//
//   * W is the MMA's M operand: one 128-row vocab tile per accumulator, its
//     K-slices (64 hidden elements, 16 KB) streamed by TMA through a ring of
//     shared-memory stages; the packed rows are the N operand (N <= 256).
//   * Persistent CTAs: rows are split into G groups of <= 256 (G = 1 for
//     M <= 256); the vocab tiles into R = gridDim / G contiguous ranges; CTA
//     (group, range) streams its range once.
//   * Warp roles: warp 0 issues TMA, warp 1 issues tcgen05.mma into one of
//     two TMEM accumulators (128 lanes x 256 fp32 columns each), warps 2-5
//     drain the other accumulator: per column (= packed row) a warp-wide
//     max / argmax / sum of exp over its 32 vocab lanes, folded into a
//     running (max, sum, argmax) that lane (column mod 32) keeps.
//   * At the end the 4 epilogue warps combine through shared memory and the
//     CTA writes one (max, sum, argmax) partial per row of its group.
#include "lmhead_common.cuh"

namespace bd {
namespace {

using lmh::kKStage;
using lmh::kVTile;
using lmh::kWBytes;
using lmh::round16;

constexpr int kThreads = 192;  // 6 warps
constexpr int kMaxN = 256;     // packed rows per group (MMA N)
constexpr int kMaxStages = 12;
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemBytes = 192 * 1024;  // + ~29 KB static stays under 227 KB

struct SelectTcArgs {
  const uint32_t* masked;  // [batch] masked-position bits: M = total popcount of the scored bits
  int batch;
  int S, active;           // sub-block size; active-only scoring (scored_bits)
  int seq_words;           // > 0: cross-entropy rows; bit 0 of every seq_words-th word is not scored
  int H, V;
  int rows_alloc;
  int part_stride;  // partials are [row][part]
  float* pm;
  float* ps;
  int32_t* pa;
  int32_t* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    lmhead_tc_kernel(const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_w16,
                     const __grid_constant__ CUtensorMap tm_rows, SelectTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2];
  __shared__ uint32_t tmem_slot;
  __shared__ float red_m[4][kMaxN];
  __shared__ float red_s[4][kMaxN];
  __shared__ int red_a[4][kMaxN];
  __shared__ float xpose[4][32 * 33];  // per epilogue warp: a 32 x 32 chunk, transposed

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // M, the number of packed rows, from the caller's mask bits (the gather
  // kernel, which packs the rows, counts the same bits), so the CTA's share
  // of the work is known before the gather kernel completes.
  {
    int acc = 0;
    for (int x = threadIdx.x; x < a.batch; x += blockDim.x)
      acc += __popc(a.seq_words > 0 ? ce_scored_bits(a.masked[x], x, a.seq_words)
                                    : scored_bits(a.masked[x], a.S, a.active));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) red_a[0][warp] = acc;
    __syncthreads();
  }
  int M = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) M += red_a[0][w];
  __syncthreads();
  const int G = (M + kMaxN - 1) / kMaxN;
  const int R = M > 0 ? gridDim.x / G : 1;
  const int group = blockIdx.x / R, range = blockIdx.x % R;
  const int Ng = M > 0 ? round16((M + G - 1) / G) : 0;
  const int row0 = group * Ng;
  const int rows_here = min(Ng, M - row0);
  if (M <= 0 || group >= G || rows_here <= 0) {
    griddep_wait();  // completes only after the gather kernel
    return;
  }
  const int N = round16(rows_here);
  // Balanced vocab ranges in units of 16 rows: [v0, v1), split into 128-row
  // tiles.  The first tile takes the remainder (rem rows, loaded in 16-row
  // boxes when short), so that its small loads overlap the full tiles
  // streaming behind it instead of trailing at the end of the range.
  const int n_u = (a.V + 15) / 16;
  const int v0 = 16 * static_cast<int>(static_cast<long long>(range) * n_u / R);
  const int v1 = min(a.V, 16 * static_cast<int>(static_cast<long long>(range + 1) * n_u / R));
  const int n_t = (v1 - v0 + kVTile - 1) / kVTile;
  const int rem = v1 - v0 - (n_t - 1) * kVTile;  // rows of tile 0 (1..128 when n_t > 0)
  auto tile_start = [&](int it) { return it == 0 ? v0 : v0 + rem + (it - 1) * kVTile; };
  auto tile_rows = [&](int it) { return it == 0 ? rem : kVTile; };
  const int n_k = (a.H + kKStage - 1) / kKStage;
  const int b_bytes = N * kKStage * 2;
  const int stage_bytes = (kWBytes + b_bytes + 1023) & ~1023;
  int n_stages = (kSmemBytes - 1024) / stage_bytes;
  n_stages = n_stages > kMaxStages ? kMaxStages : n_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < n_stages; ++s) {
      tc::mbar_init(&full_bar[s], 1);
      tc::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull_bar[b], 1);
      tc::mbar_init(&tempty_bar[b], 4);
    }
    tc::fence_barrier_init();
    tc::fence_proxy_async();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  griddep_launch_dependents();
  if (warp != 0) griddep_wait();  // status and partials are written after the gather kernel

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_w);
      tc::prefetch_tmap(&tm_w16);
      tc::prefetch_tmap(&tm_rows);
      const uint64_t pol_w = tc::policy_evict_first();
      const uint64_t pol_r = tc::policy_evict_last();
      // Stage i of the flat (vocab tile, K-slice) sequence: its W slice (a
      // short last tile in 16-row boxes; rows past it are never used) and
      // its packed-row slice.
      auto w_bytes = [&](int i) {
        const int nw = tile_rows(i / n_k);
        return nw == kVTile ? kWBytes : (nw + 15) / 16 * 2048;
      };
      auto load_w = [&](int i, uint8_t* st, uint64_t* bar) {
        const int vt = tile_start(i / n_k), kb = i % n_k;
        if (w_bytes(i) == kWBytes) {
          tc::tma_load_2d(st, &tm_w, bar, kb * kKStage, vt, pol_w);
        } else {
          for (int j = 0; j < w_bytes(i) / 2048; ++j)
            tc::tma_load_2d(st + j * 2048, &tm_w16, bar, kb * kKStage, vt + 16 * j, pol_w);
        }
      };
      auto load_rows = [&](int i, uint8_t* st, uint64_t* bar) {
        for (int j = 0; j < N / 16; ++j)
          tc::tma_load_2d(st + kWBytes + j * 2048, &tm_rows, bar, (i % n_k) * kKStage,
                          row0 + 16 * j, pol_r);
      };
      // W does not depend on the gather kernel: fill the (free) ring with W
      // slices first, then add the packed rows once the gather completes.
      const int n_total = n_t * n_k;
      const int n_pre = min(n_stages, n_total);
      for (int i = 0; i < n_pre; ++i) {
        uint8_t* st = smem + static_cast<size_t>(i) * stage_bytes;
        tc::mbar_arrive_expect_tx(&full_bar[i], w_bytes(i) + b_bytes);
        load_w(i, st, &full_bar[i]);
      }
      griddep_wait();
      for (int i = 0; i < n_pre; ++i)
        load_rows(i, smem + static_cast<size_t>(i) * stage_bytes, &full_bar[i]);
      int s = n_pre % n_stages;
      uint32_t ph = n_pre / n_stages;
      for (int i = n_pre; i < n_total; ++i) {
        if (!tc::mbar_wait(&empty_bar[s], ph ^ 1, a.status)) break;
        uint8_t* st = smem + static_cast<size_t>(s) * stage_bytes;
        tc::mbar_arrive_expect_tx(&full_bar[s], w_bytes(i) + b_bytes);
        load_w(i, st, &full_bar[s]);
        load_rows(i, st, &full_bar[s]);
        if (++s == n_stages) { s = 0; ph ^= 1; }
      }
    }
    __syncwarp();
    if (lane != 0) griddep_wait();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kVTile, N);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = 0; it < n_t && ok; ++it) {
        const int b = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!tc::mbar_wait(&tempty_bar[b], tph ^ 1, a.status)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + b * kMaxN;
        for (int kb = 0; kb < n_k; ++kb) {
          if (!tc::mbar_wait(&full_bar[s], ph, a.status)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = tc::smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
          const uint32_t sb = sa + kWBytes;
#pragma unroll
          for (int kk = 0; kk < kKStage / 16; ++kk)
            tc::mma_bf16_ss(d, tc::sdesc_kmajor_sw128(sa + kk * 32),
                            tc::sdesc_kmajor_sw128(sb + kk * 32), idesc, (kb | kk) != 0);
          tc::mma_commit(&empty_bar[s]);
          if (++s == n_stages) { s = 0; ph ^= 1; }
        }
        tc::mma_commit(&tfull_bar[b]);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    lmh::Run run[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) run[c] = lmh::run_empty();
    const int n_chunks = N / 32 + ((N % 32) ? 1 : 0);
    bool ok = true;
    for (int it = 0; it < n_t && ok; ++it) {
      const int b = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!tc::mbar_wait_warp(&tfull_bar[b], tph, a.status)) { ok = false; break; }
      tc::tc_fence_after();
      const int vbase = tile_start(it) + q * 32;  // vocab row of this warp's lane 0
      const int vend = tile_start(it) + tile_rows(it);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c < n_chunks)
          lmh::fold_chunk(tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kMaxN + c * 32,
                          xpose[q], lane, vbase, vend, run[c]);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty_bar[b]);
    }
    // combine the 4 lane quarters through shared memory
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int col = c * 32 + lane;
      if (col < N) {
        red_m[q][col] = run[c].m;
        red_s[q][col] = run[c].s;
        red_a[q][col] = run[c].a;
      }
    }
    tc::named_bar_sync(1, 128);
    const int et = threadIdx.x - 64;
    for (int col = et; col < rows_here; col += 128) {
      Stat st = stat_empty();
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) st = stat_combine(st, Stat{red_m[qq][col], red_s[qq][col], red_a[qq][col]});
      const size_t idx = static_cast<size_t>(row0 + col) * a.part_stride + range;
      a.pm[idx] = st.m;
      a.ps[idx] = st.s;
      a.pa[idx] = st.a;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

int lmhead_tc_grid() { return lmh::sm_count(); }

cudaError_t launch_lmhead_tc(const void* rows, const void* w, const uint32_t* masked, int batch,
                             int S, int active, int H, int V, int rows_alloc, int part_stride,
                             float* pm, float* ps, int32_t* pa, int32_t* status, cudaStream_t st,
                             int seq_words) {
  CUtensorMap tm_w, tm_w16, tm_rows;
  if (!lmh::make_tmap_2d(&tm_w, w, static_cast<uint64_t>(V), static_cast<uint64_t>(H), kVTile) ||
      !lmh::make_tmap_2d(&tm_w16, w, static_cast<uint64_t>(V), static_cast<uint64_t>(H), 16) ||
      !lmh::make_tmap_2d(&tm_rows, rows, static_cast<uint64_t>(rows_alloc), static_cast<uint64_t>(H),
                    16))
    return cudaErrorInvalidValue;
  SelectTcArgs a{masked, batch, S, active, seq_words, H, V, rows_alloc, part_stride, pm, ps, pa,
                 status};
  cudaFuncSetAttribute(lmhead_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kSmemBytes + 1024);
  const cudaError_t e = launch_pdl(lmhead_tc_kernel, dim3(lmhead_tc_grid()), dim3(kThreads),
                                   kSmemBytes + 1024, st, tm_w, tm_w16, tm_rows, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd
