// LM-head statistics for many packed rows at once (the cross-entropy of a
// training batch: thousands of rows), on the 5th-generation tensor cores.
//
// The LM head of bd_confidence_select makes W the MMA's 128-row M operand
// and the few packed rows its N operand, re-reading every row for every
// vocab tile; with thousands of rows that re-read dominates.  Here the rows
// are the M operand and W the N operand:
//
//   * unit = (row pair rp, vocab range v): 2 x 128 packed rows against the
//     256-row W tiles of one of R contiguous vocab ranges.  Per 64-element
//     K-slice a stage holds both row tiles (2 x 16 KB) and one W tile
//     (32 KB): 64 KB for two 128 x 256 x 64 products.
//   * persistent CTAs, one per SM, take units u = blockIdx.x + k * gridDim.x
//     with rp fastest, so the CTAs running at one time stream the same few
//     vocab ranges: W comes from HBM a few times in all (CTAs drift apart
//     over a range), the rows (they fit in L2) from L2.
//   * warp 0 streams the stages by TMA (3 stages), warp 1 issues tcgen05.mma
//     into two 256-column TMEM accumulators (one per row tile), warps 2-17
//     each drain 32 rows x 128 columns after a W tile; a thread owns one row,
//     so the fold into its running (max, sum exp) needs no shuffles.  The
//     accumulators are not double-buffered (2 x 256 columns fill TMEM): the
//     MMA waits for each drain, so the drain is spread over 16 warps with
//     the next TMEM load in flight during each fold.
//   * per unit, each row gets two (max, sum exp) partials, one per column
//     half: [row][2 R].
#include "lmhead_common.cuh"

namespace bd {
namespace {

constexpr int kThreads = 576;                 // 18 warps
constexpr int kRowTile = 128;                 // MMA M
constexpr int kWTile = 256;                   // MMA N: vocab rows per W tile
constexpr int kK = 64;                        // hidden elements per stage
constexpr int kRowBytes = kRowTile * kK * 2;  // 16 KB
constexpr int kWTileBytes = kWTile * kK * 2;  // 32 KB
constexpr int kStageBytes = 2 * kRowBytes + kWTileBytes;
constexpr int kStages = 3;
constexpr int kSmemBytes = kStages * kStageBytes + 1024;  // + alignment slack
constexpr uint32_t kTmemCols = 512;

struct RowsArgs {
  const uint32_t* masked;  // mask words of the batch (ce_scored_bits)
  int n_words, seq_words;
  int H, V;
  int R;                   // vocab ranges (2 R partials per row)
  float* pm;               // [row][2 R]
  float* ps;
  int32_t* status;
};

// Folds 32 logits (the first n valid; kFull: all 32) into a running
// (max, sum exp).
template <bool kFull>
__device__ __forceinline__ void fold32(const uint32_t (&r)[32], int n, float& run_m,
                                       float& run_s) {
  float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float x = (kFull || i < n) ? __uint_as_float(r[i]) : -INFINITY;
    mk[i & 3] = fmaxf(mk[i & 3], x);
  }
  const float m_new = fmaxf(run_m, fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])));
  if (m_new == -INFINITY) return;
  const float mls = m_new * kLog2e;
  float sk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (kFull || i < n) {
      const float y = fmaf(__uint_as_float(r[i]), kLog2e, -mls);
      // one exponential in four on the FMA pipe, the rest on MUFU
      sk[i & 3] += (i & 3) == 3 ? poly_exp2(y) : fast_exp2(y);
    }
  }
  run_s = run_s * fast_exp2((run_m - m_new) * kLog2e) + ((sk[0] + sk[1]) + (sk[2] + sk[3]));
  run_m = m_new;
}

__global__ void __launch_bounds__(kThreads, 1)
    lmhead_rows_kernel(const __grid_constant__ CUtensorMap tm_rows,
                       const __grid_constant__ CUtensorMap tm_w, RowsArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], tfull_bar, tempty_bar, done_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int red[kThreads / 32];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // M from the mask words (inputs of the call, complete before the gather
  // kernel let this one start); the gather kernel counts the same bits
  {
    int acc = 0;
    for (int x = threadIdx.x; x < a.n_words; x += blockDim.x)
      acc += __popc(ce_scored_bits(a.masked[x], x, a.seq_words));
    acc = __reduce_add_sync(0xffffffffu, acc);
    if (lane == 0) red[warp] = acc;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full_bar[s], 1);
      tc::mbar_init(&empty_bar[s], 1);
    }
    tc::mbar_init(&tfull_bar, 1);
    tc::mbar_init(&tempty_bar, 16);
    tc::mbar_init(&done_bar, 1);
    tc::fence_barrier_init();
    tc::fence_proxy_async();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  int M = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) M += red[w];
  const int RP = (M + 2 * kRowTile - 1) / (2 * kRowTile);
  const int n_units = RP * a.R;
  const int n_wt = (a.V + kWTile - 1) / kWTile;
  const int n_k = (a.H + kK - 1) / kK;
  // W tiles [wt0, wt1) of vocab range v
  auto range = [&](int v, int& wt0, int& wt1) {
    wt0 = static_cast<int>(static_cast<long long>(v) * n_wt / a.R);
    wt1 = static_cast<int>(static_cast<long long>(v + 1) * n_wt / a.R);
  };
  griddep_launch_dependents();
  griddep_wait();  // the packed rows and the status word of the gather kernel

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_rows);
      tc::prefetch_tmap(&tm_w);
      const uint64_t pol_w = tc::policy_evict_first();
      const uint64_t pol_r = tc::policy_evict_last();
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int v = u / RP, row0 = (u % RP) * 2 * kRowTile;
        int wt0, wt1;
        range(v, wt0, wt1);
        for (int wt = wt0; wt < wt1 && ok; ++wt) {
          for (int kb = 0; kb < n_k; ++kb) {
            if (!tc::mbar_wait(&empty_bar[s], ph ^ 1, a.status)) { ok = false; break; }
            uint8_t* st = smem + s * kStageBytes;
            tc::mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
            tc::tma_load_2d(st, &tm_rows, &full_bar[s], kb * kK, row0, pol_r);
            tc::tma_load_2d(st + kRowBytes, &tm_rows, &full_bar[s], kb * kK, row0 + kRowTile,
                            pol_r);
            tc::tma_load_2d(st + 2 * kRowBytes, &tm_w, &full_bar[s], kb * kK, wt * kWTile, pol_w);
            ++issued;
            if (++s == kStages) { s = 0; ph ^= 1; }
          }
        }
      }
      // every copy this thread started has landed before the CTA exits
      // (immediate on the normal path: the MMA issuer consumed them all)
      for (int i = 1; i <= kStages && i <= issued; ++i) {
        const int j = issued - i;
        tc::mbar_wait(&full_bar[j % kStages], (j / kStages) & 1, a.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kRowTile, kWTile);
      int s = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int wt0, wt1;
        range(u / RP, wt0, wt1);
        for (int wt = wt0; wt < wt1 && ok; ++wt, ++it) {
          // the accumulators of the previous W tile have been drained
          if (!tc::mbar_wait(&tempty_bar, (it & 1) ^ 1, a.status)) { ok = false; break; }
          tc::tc_fence_after();
          for (int kb = 0; kb < n_k; ++kb) {
            if (!tc::mbar_wait(&full_bar[s], ph, a.status)) { ok = false; break; }
            tc::tc_fence_after();
            const uint32_t sa = tc::smem_u32(smem + s * kStageBytes);
            const uint32_t sw = sa + 2 * kRowBytes;
#pragma unroll
            for (int kk = 0; kk < kK / 16; ++kk) {
              const uint64_t bw = tc::sdesc_kmajor_sw128(sw + kk * 32);
              const uint32_t acc = (kb | kk) != 0;
              tc::mma_bf16_ss(tmem, tc::sdesc_kmajor_sw128(sa + kk * 32), bw, idesc, acc);
              tc::mma_bf16_ss(tmem + kWTile, tc::sdesc_kmajor_sw128(sa + kRowBytes + kk * 32), bw,
                              idesc, acc);
            }
            tc::mma_commit(&empty_bar[s]);
            if (++s == kStages) { s = 0; ph ^= 1; }
          }
          if (ok) tc::mma_commit(&tfull_bar);
        }
      }
      // every MMA this thread issued has completed before TMEM is released
      tc::mma_commit(&done_bar);
      tc::mbar_wait(&done_bar, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    // warps 2..17 (e = warp - 2): row tile tt, column half hf of the W tile,
    // TMEM lane quarter q (= warp % 4, the lanes this warp may access); one
    // row per thread, four 32-column chunks per W tile, the load of the next
    // chunk in flight while this one is folded
    const int e = warp - 2, tt = (e >> 2) & 1, hf = e >> 3, q = warp & 3;
    const uint32_t tbase =
        tmem + (static_cast<uint32_t>(q * 32) << 16) + tt * kWTile + hf * (kWTile / 2);
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int v = u / RP;
      const int row = (u % RP) * 2 * kRowTile + tt * kRowTile + q * 32 + lane;
      int wt0, wt1;
      range(v, wt0, wt1);
      float run_m = -INFINITY, run_s = 0.f;
      for (int wt = wt0; wt < wt1; ++wt, ++it) {
        if (!tc::mbar_wait_warp(&tfull_bar, it & 1, a.status)) { ok = false; break; }
        tc::tc_fence_after();
        // valid columns of this warp's half of the W tile (warp-uniform)
        const int lim = min(kWTile, a.V - wt * kWTile) - hf * (kWTile / 2);
        const int nc = lim <= 0 ? 0 : min(4, (lim + 31) / 32);
        uint32_t rb[2][32];
        if (nc > 0) tc::tmem_ld_32x32b_x32(tbase, rb[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < nc) {
            tc::tmem_ld_wait(rb[c & 1]);
            if (c + 1 < nc) tc::tmem_ld_32x32b_x32(tbase + (c + 1) * 32, rb[(c + 1) & 1]);
            if (lim >= (c + 1) * 32)
              fold32<true>(rb[c & 1], 32, run_m, run_s);
            else
              fold32<false>(rb[c & 1], lim - c * 32, run_m, run_s);
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty_bar);
      }
      if (ok && row < M) {
        a.pm[static_cast<size_t>(row) * 2 * a.R + 2 * v + hf] = run_m;
        a.ps[static_cast<size_t>(row) * 2 * a.R + 2 * v + hf] = run_s;
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// Partials per row = 2 x the vocab ranges.
int lmhead_rows_ranges(int vocab) {
  // about 8 W tiles per unit, at most 64 partials per row
  const int n_wt = (vocab + kWTile - 1) / kWTile;
  const int R = n_wt / 8;
  return R < 1 ? 1 : (R > 64 ? 64 : R);
}

cudaError_t launch_lmhead_rows(const void* rows, const void* w, const uint32_t* masked,
                               int n_words, int seq_words, int H, int V, int rows_alloc, int R,
                               float* pm, float* ps, int32_t* status, cudaStream_t st) {
  if (rows_alloc % (2 * kRowTile) != 0 || H % 8 != 0) return cudaErrorInvalidValue;
  CUtensorMap tm_rows, tm_w;
  if (!lmh::make_tmap_2d(&tm_rows, rows, static_cast<uint64_t>(rows_alloc),
                         static_cast<uint64_t>(H), kRowTile) ||
      !lmh::make_tmap_2d(&tm_w, w, static_cast<uint64_t>(V), static_cast<uint64_t>(H), kWTile))
    return cudaErrorInvalidValue;
  RowsArgs a{masked, n_words, seq_words, H, V, R, pm, ps, status};
  cudaError_t e = cudaFuncSetAttribute(lmhead_rows_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(lmhead_rows_kernel, dim3(lmh::sm_count()), dim3(kThreads), kSmemBytes, st,
                 tm_rows, tm_w, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd
