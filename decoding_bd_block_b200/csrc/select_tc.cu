// LM-head statistics on the 5th-generation tensor cores (bf16 in, fp32
// accumulate), for bd_confidence_select with more than one sequence.
//
// Each packed row r (the hidden row that predicts one masked position) needs
// max_v l, sum_v exp(l - max) and argmax_v of l = row . W[v] over the whole
// vocabulary ("Fast-dLLM v2: Efficient Block-Diffusion LLM", key design 3:
// confidence of a masked token; Fast-dLLM v1 article, core technique 2).
// The logits never leave the chip:
//
//   * The packed rows are the MMA's M operand: a row group of up to 256 rows
//     is one or two 128-row tiles, each with its own TMEM accumulator; W is
//     the N operand, in tiles of up to 256 vocab rows.  A stage of the
//     shared-memory ring holds one 64-element K-slice of the row tiles and
//     of the W tile, so every byte of rows read from L2 serves up to 256
//     vocab rows (the W-as-M arrangement re-read the rows for every 128).
//   * Persistent CTAs: rows are split into G = ceil(M / 256) groups, the
//     vocabulary into R = gridDim / G contiguous ranges; CTA (group, range)
//     streams its range once, in equal tiles of TR rows (TR a multiple of
//     16, the fewest tiles that cover the range), so no short tail tile
//     costs a full pass over the rows.
//   * The stream is bound by the bytes each SM has in flight (a stage's
//     loads take ~2 us to land whether they come from HBM or L2), so the
//     tile height is capped to keep four stages in shared memory, and each
//     row tile's box is only as high as its valid rows (rows past them are
//     stale shared memory: their accumulator lanes are never read).
//   * Each stage is two or three TMA boxes (the row tiles and one W box):
//     the TMA cost grows with the number of boxes, so every box matches its
//     tile exactly, from sets of tensor maps with box heights 16, 32, ...,
//     passed by value.
//   * Warp roles: warp 0 issues TMA, warp 1 issues tcgen05.mma, warps 2-17
//     drain the accumulators: warp (tile m, column half hf, lane quarter q)
//     owns rows m * 128 + 32 q .. + 31, one row per thread, and folds its
//     half of the row's columns (vocab entries), 32 at a time, into a
//     running (max, sum exp, argmax) with plain per-thread arithmetic.  Two
//     row tiles fill TMEM (2 x 256
//     columns), so then the MMA waits for each drain; a single row tile is
//     double-buffered.
//   * At the end the two column halves of each row are combined and
//     every CTA writes one (max, sum, argmax) partial per row of its group.
#include "lmhead_common.cuh"

namespace bd {
namespace {

constexpr int kThreads = 576;                   // 18 warps
constexpr int kEpiWarps = 16;
constexpr int kRowTile = 128;                   // MMA M: packed rows per accumulator
constexpr int kGroupRows = 2 * kRowTile;        // packed rows per row group
constexpr int kMaxWTile = 256;                  // MMA N: vocab rows per W tile
constexpr int kK = 64;                          // hidden elements per stage (128-byte rows)
constexpr int kRowLine = kK * 2;                // bytes of one row's K-slice
constexpr int kRowTileBytes = kRowTile * kRowLine;  // 16 KB
constexpr int kStagesWanted = 4;
constexpr int kMaxStages = 8;
constexpr int kSmemBytes = 224 * 1024;          // + 1 KB alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;              // TMEM columns per accumulator
constexpr int kNumWMaps = kMaxWTile / 16;
constexpr int kNumRowMaps = kRowTile / 16;

// Tensor maps with box heights 16 (i + 1): W tiles and row tiles.
struct BoxMaps {
  CUtensorMap w[kNumWMaps];
  CUtensorMap rows[kNumRowMaps];
};

struct SelectTcArgs {
  const uint32_t* masked;  // [batch] masked-position bits: M = total popcount of the scored bits
  int batch;
  int S, active;           // sub-block size; active-only scoring (scored_bits)
  int seq_words;           // > 0: cross-entropy rows; bit 0 of every seq_words-th word is not scored
  int H, V;
  int part_stride;         // partials are [row][part]
  float* pm;
  float* ps;
  int32_t* pa;
  int32_t* status;
};


// Folds 32 logits of one row -- vocab entries vbase .. vbase + 31, the first
// n of them valid (kFull: all 32) -- into the thread's running statistics.
// The chunks of one thread arrive in increasing vocab order, so an equal
// maximum later never replaces the running one (ties keep the lowest index).
template <bool kFull>
__device__ __forceinline__ void fold_row32(const uint32_t (&r)[32], int n, int vbase,
                                           lmh::Run& run) {
  float x[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = (kFull || i < n) ? __uint_as_float(r[i]) : -INFINITY;
  float mk[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) mk[k] = tc::fmax3(x[8 * k], x[8 * k + 1], x[8 * k + 2]);
#pragma unroll
  for (int k = 0; k < 4; ++k) mk[k] = tc::fmax3(mk[k], x[8 * k + 3], x[8 * k + 4]);
#pragma unroll
  for (int k = 0; k < 4; ++k) mk[k] = tc::fmax3(mk[k], x[8 * k + 5], x[8 * k + 6]);
#pragma unroll
  for (int k = 0; k < 4; ++k) mk[k] = fmaxf(mk[k], x[8 * k + 7]);
  const float mx = fmaxf(tc::fmax3(mk[0], mk[1], mk[2]), mk[3]);
  if (mx == -INFINITY) return;
  const float m_new = fmaxf(run.m, mx);
  if (mx > run.m) {  // a new running maximum: its lowest index in the chunk
    // four independent chains (indices k mod 4), then the lowest of them
    int ak[4] = {32, 32, 32, 32};
#pragma unroll
    for (int i = 31; i >= 0; --i) ak[i & 3] = x[i] == mx ? i : ak[i & 3];
    run.a = vbase + min(min(ak[0], ak[1]), min(ak[2], ak[3]));
  }
  const float2 l2 = make_float2(kLog2e, kLog2e);
  const float2 nm = make_float2(-m_new * kLog2e, -m_new * kLog2e);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    // paired fp32 arithmetic; one pair in four on the FMA pipe, the rest on MUFU
    const float2 y = ffma2(make_float2(x[2 * k], x[2 * k + 1]), l2, nm);
    const float2 e = (k & 3) == 3 ? poly_exp2x2(y) : make_float2(fast_exp2(y.x), fast_exp2(y.y));
    acc[k & 1] = fadd2(acc[k & 1], e);
  }
  const float e = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
  run.s = (mx > run.m ? run.s * fast_exp2((run.m - m_new) * kLog2e) : run.s) + e;
  run.m = m_new;
}

__global__ void __launch_bounds__(kThreads, 1)
    lmhead_tc_kernel(const __grid_constant__ BoxMaps maps, SelectTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2], done_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int red[kThreads / 32];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // M, the number of packed rows, from the caller's mask bits (the gather
  // kernel, which packs the rows, counts the same bits), so the CTA's share
  // of the work is known before the gather kernel completes.
  {
    int acc = 0;
    for (int x = threadIdx.x; x < a.batch; x += blockDim.x)
      acc += __popc(a.seq_words > 0 ? ce_scored_bits(a.masked[x], x, a.seq_words)
                                    : scored_bits(a.masked[x], a.S, a.active));
    acc = __reduce_add_sync(0xffffffffu, acc);
    if (lane == 0) red[warp] = acc;
    __syncthreads();
  }
  int M = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) M += red[w];
  const int G = (M + kGroupRows - 1) / kGroupRows;
  const int R = M > 0 ? static_cast<int>(gridDim.x) / G : 1;
  const int group = blockIdx.x / R, range = blockIdx.x % R;
  const int row0 = group * kGroupRows;
  if (M <= 0 || group >= G) {
    griddep_wait();  // completes only after the gather kernel
    return;
  }
  const int rows_here = min(kGroupRows, M - row0);
  const int mt = (rows_here + kRowTile - 1) / kRowTile;  // row tiles: 1 or 2
  // box height of row tile m: its valid rows, rounded up to 16
  auto rbox = [&](int m) { return lmh::round16(min(kRowTile, rows_here - m * kRowTile)); };
  const int r_bytes = (rbox(0) + (mt == 2 ? rbox(1) : 0)) * kRowLine;
  // Vocab range [v0, v1) in units of 16 rows, cut into n_t tiles of TR rows
  // (the last one may be shorter; rows past v1 are loaded but not used).
  // TR is capped so that kStagesWanted stages fit in shared memory.
  const int n_u = (a.V + 15) / 16;
  const int v0 = 16 * static_cast<int>(static_cast<long long>(range) * n_u / R);
  const int v1 = min(a.V, 16 * static_cast<int>(static_cast<long long>(range + 1) * n_u / R));
  const int len = v1 - v0;
  const int tr_cap =
      max(16, min(kMaxWTile, ((kSmemBytes / kStagesWanted - r_bytes) / kRowLine) / 16 * 16));
  const int n_t = (len + tr_cap - 1) / tr_cap;
  const int TR = n_t > 0 ? lmh::round16((len + n_t - 1) / n_t) : 16;
  const CUtensorMap* tm_w = &maps.w[TR / 16 - 1];
  auto tile_start = [&](int it) { return v0 + it * TR; };
  auto tile_rows = [&](int it) { return min(TR, v1 - tile_start(it)); };
  const int n_k = (a.H + kK - 1) / kK;
  const int w_bytes = TR * kRowLine;
  // Stage layout: row tile 0 | row tile 1 (only the boxes' rows are
  // loaded) | W tile, each part 1024-byte aligned for the swizzle atoms.
  const int r1_off = rbox(0) * kRowLine;  // a multiple of 2048
  const int w_off = mt == 2 ? r1_off + rbox(1) * kRowLine : r1_off;
  const int stage_bytes = (w_off + w_bytes + 1023) & ~1023;
  // The MMA reads each row tile at its full 128 rows, past a short box into
  // the rest of the stage (lanes that are never read back); keep that read
  // of the last stage inside the allocation too.
  const int a_end = (mt - 1) * r1_off + kRowTileBytes;
  const int overrun = a_end > stage_bytes ? a_end - stage_bytes : 0;
  int n_stages = (kSmemBytes - overrun) / stage_bytes;
  n_stages = n_stages > kMaxStages ? kMaxStages : n_stages;
  const int load_tx = r_bytes + w_bytes;  // bytes the boxes of one stage bring
  // Accumulator of row tile m for W tile it: two row tiles fill TMEM (one
  // buffer); one row tile alternates between two buffers.
  const int n_buf = mt == 2 ? 1 : 2;
  auto buf_of = [&](int it) { return n_buf == 1 ? 0 : (it & 1); };
  auto use_of = [&](int it) { return n_buf == 1 ? it : (it >> 1); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < n_stages; ++s) {
      tc::mbar_init(&full_bar[s], 1);
      tc::mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull_bar[b], 1);
      tc::mbar_init(&tempty_bar[b], 8 * mt);
    }
    tc::mbar_init(&done_bar, 1);
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
      tc::prefetch_tmap(tm_w);
      for (int m = 0; m < mt; ++m) tc::prefetch_tmap(&maps.rows[rbox(m) / 16 - 1]);
      const uint64_t pol_w = tc::policy_evict_first();
      const uint64_t pol_r = tc::policy_evict_last();
      // Stage i of the flat (W tile, K-slice) sequence.
      auto load_w = [&](int i, uint8_t* st, uint64_t* bar) {
        tc::tma_load_2d(st + w_off, tm_w, bar, (i % n_k) * kK, tile_start(i / n_k), pol_w);
      };
      auto load_rows = [&](int i, uint8_t* st, uint64_t* bar) {
        for (int m = 0; m < mt; ++m)
          tc::tma_load_2d(st + m * r1_off, &maps.rows[rbox(m) / 16 - 1], bar, (i % n_k) * kK,
                          row0 + m * kRowTile, pol_r);
      };
      // W does not depend on the gather kernel: fill the (free) ring with W
      // slices first, then add the packed rows once the gather completes.
      const int n_total = n_t * n_k;
      const int n_pre = min(n_stages, n_total);
      for (int i = 0; i < n_pre; ++i) {
        uint8_t* st = smem + static_cast<size_t>(i) * stage_bytes;
        tc::mbar_arrive_expect_tx(&full_bar[i], load_tx);
        load_w(i, st, &full_bar[i]);
      }
      griddep_wait();
      for (int i = 0; i < n_pre; ++i)
        load_rows(i, smem + static_cast<size_t>(i) * stage_bytes, &full_bar[i]);
      int s = n_pre % n_stages, issued = n_pre;
      uint32_t ph = n_pre / n_stages;
      for (int i = n_pre; i < n_total; ++i) {
        if (!tc::mbar_wait(&empty_bar[s], ph ^ 1, a.status)) break;
        uint8_t* st = smem + static_cast<size_t>(s) * stage_bytes;
        tc::mbar_arrive_expect_tx(&full_bar[s], load_tx);
        load_w(i, st, &full_bar[s]);
        load_rows(i, st, &full_bar[s]);
        ++issued;
        if (++s == n_stages) { s = 0; ph ^= 1; }
      }
      // every copy this thread started has landed before the CTA exits
      // (immediate on the normal path: the MMA issuer consumed them all)
      for (int k = 1; k <= n_stages && k <= issued; ++k) {
        const int j = issued - k;
        tc::mbar_wait(&full_bar[j % n_stages], (j / n_stages) & 1, a.status);
      }
    }
    __syncwarp();
    if (lane != 0) griddep_wait();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kRowTile, TR);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = 0; it < n_t && ok; ++it) {
        const int b = buf_of(it);
        // the accumulator's previous use has been drained
        if (!tc::mbar_wait(&tempty_bar[b], (use_of(it) & 1) ^ 1, a.status)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + b * kAccCols;
        for (int kb = 0; kb < n_k; ++kb) {
          if (!tc::mbar_wait(&full_bar[s], ph, a.status)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = tc::smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
#pragma unroll
          for (int kk = 0; kk < kK / 16; ++kk) {
            const uint64_t bw = tc::sdesc_kmajor_sw128(sa + w_off + kk * 32);
            const uint32_t acc = (kb | kk) != 0;
            for (int m = 0; m < mt; ++m)
              tc::mma_bf16_ss(d + m * kAccCols, tc::sdesc_kmajor_sw128(sa + m * r1_off + kk * 32),
                              bw, idesc, acc);
          }
          tc::mma_commit(&empty_bar[s]);
          if (++s == n_stages) { s = 0; ph ^= 1; }
        }
        if (ok) tc::mma_commit(&tfull_bar[b]);
      }
      // every MMA this thread issued has completed before TMEM is released
      tc::mma_commit(&done_bar);
      tc::mbar_wait(&done_bar, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    // warps 2..17: row tile m, column half hf, TMEM lane quarter q (= warp
    // % 4, the lanes this warp may access); thread = one packed row
    const int e = warp - 2, m = (e >> 2) & 1, hf = e >> 3, q = warp & 3;
    const int lrow = m * kRowTile + q * 32 + lane;  // row within the group
    lmh::Run run = lmh::run_empty();
    bool ok = m < mt;
    for (int it = 0; it < n_t && ok; ++it) {
      const int b = buf_of(it);
      if (!tc::mbar_wait_warp(&tfull_bar[b], use_of(it) & 1, a.status)) { ok = false; break; }
      tc::tc_fence_after();
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * kAccCols +
                             (n_buf == 1 ? m * kAccCols : 0);
      // this warp's columns: the first or the second half of the tile's
      // valid columns (split at a multiple of 16), in 32-column chunks
      const int nv = tile_rows(it);  // valid columns (warp-uniform)
      const int mid = min(nv, lmh::round16((nv + 1) / 2));
      const int c0 = hf ? mid : 0, c1 = hf ? nv : mid;
      const int vb = tile_start(it);
#pragma unroll 1
      for (int c = c0; c < c1; c += 32) {
        uint32_t rb[32];
        tc::tmem_ld_32x32b_x32(tbase + c, rb);
        tc::tmem_ld_wait(rb);
        if (c1 - c >= 32)
          fold_row32<true>(rb, 32, vb + c, run);
        else
          fold_row32<false>(rb, c1 - c, vb + c, run);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty_bar[b]);
    }
    // Combine the two column halves of each row.  The shared-memory
    // ring is free by now: every stage's copies have landed and the MMAs
    // that read them completed before the last accumulator was full.
    float* cm = reinterpret_cast<float*>(smem);
    float* cs = cm + kGroupRows;
    int* ca = reinterpret_cast<int*>(cs + kGroupRows);
    if (ok && hf == 1) {
      cm[lrow] = run.m;
      cs[lrow] = run.s;
      ca[lrow] = run.a;
    }
    tc::named_bar_sync(1, 32 * kEpiWarps);
    if (ok && hf == 0 && row0 + lrow < M) {
      const Stat st = stat_combine(Stat{run.m, run.s, run.a}, Stat{cm[lrow], cs[lrow], ca[lrow]});
      const size_t idx = static_cast<size_t>(row0 + lrow) * a.part_stride + range;
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
  // every row tile lies inside the packed-row buffer
  if (rows_alloc % kGroupRows != 0) return cudaErrorInvalidValue;
  BoxMaps maps;
  for (int i = 0; i < kNumWMaps; ++i)
    if (!lmh::make_tmap_2d(&maps.w[i], w, static_cast<uint64_t>(V), static_cast<uint64_t>(H),
                           16 * (i + 1)))
      return cudaErrorInvalidValue;
  for (int i = 0; i < kNumRowMaps; ++i)
    if (!lmh::make_tmap_2d(&maps.rows[i], rows, static_cast<uint64_t>(rows_alloc),
                           static_cast<uint64_t>(H), 16 * (i + 1)))
      return cudaErrorInvalidValue;
  SelectTcArgs a{masked, batch, S, active, seq_words, H, V, part_stride, pm, ps, pa, status};
  cudaError_t e = cudaFuncSetAttribute(lmhead_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes + 1024);
  if (e != cudaSuccess) return e;
  e = launch_pdl(lmhead_tc_kernel, dim3(lmhead_tc_grid()), dim3(kThreads), kSmemBytes + 1024, st,
                 maps, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd
