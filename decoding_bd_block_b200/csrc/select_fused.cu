// bd_confidence_select in ONE kernel for a single sequence: token shift, LM
// head with online softmax statistics, and the confidence-aware unmask
// ("Fast-dLLM v2: Efficient Block-Diffusion LLM", key designs 2-4; Fast-dLLM
// v1 article, confidence-aware parallel decoding).
//
// Persistent grid, one CTA per SM:
//
//   * The token shift needs no gather: the MMA's N operand is the block's 32
//     hidden rows h[0..31] followed by h_prev, fetched by TMA straight from
//     the caller's buffers (N = 48: 32 + a 16-row slot of which one row is
//     used).  Column j < 31 scores position j + 1 and column 32 position 0;
//     column 31 (the next block's first position) and 33.. are ignored.
//   * Vocab tiles of TR <= 128 rows, TR chosen by the host so that the tile
//     count is close to a multiple of the grid (151936 rows over 148 CTAs:
//     115-row tiles, 9 per CTA, instead of 1187 = 8 x 148 + 3 tiles of 128
//     that leave three CTAs a whole tile behind).  Each CTA takes tile
//     blockIdx.x, then further tiles from an atomic counter, so SMs that get
//     more HBM bandwidth take more tiles.  (A tile costs n_k ring stages
//     whatever its rows and the stream runs latency-bound on bytes in
//     flight, so tiles much smaller than 128 rows would lose bandwidth.)
//     Warp 0 streams the tile's W slices (TR x 64) with the matching 48 x 64
//     operand slice through a TMA ring; warp 1 issues tcgen05.mma (M = 128:
//     accumulator rows past TR are ignored) into one of two 64-column TMEM
//     accumulators; warps 2-5 fold the other into running (max, sum exp,
//     argmax) per column.
//   * Each CTA writes one partial per masked position; the last CTA to
//     finish (an arrival counter) merges them, applies the unmask rule and
//     zeroes the counters and the status word for the next call.
#include "lmhead_common.cuh"

namespace bd {
namespace {

using lmh::kKStage;
using lmh::kVTile;

constexpr int kThreads = 192;                         // 6 warps
constexpr int kN = 48;                                // MMA N
constexpr int kBBytes = kN * kKStage * 2;             // 6 KB operand slice
constexpr int kSmemBytes = 192 * 1024;
constexpr int kMaxStages = 12;
constexpr int kMinTileRows = 64;
constexpr uint32_t kTmemCols = 128;                   // two 64-column accumulators
constexpr int kSlots = 8;                             // published tile indices in flight
constexpr int kHpRow = 32;                            // operand row of h_prev

// Stage = W slice (TR rows x 128 bytes, rounded up to 1 KB) + operand slice.
// The MMA reads 128 rows (16 KB) of A from the stage's start, which the W
// region plus the operand slice always covers (hence W region >= 10 KB).
__host__ __device__ constexpr int stage_w_bytes(int tr) {
  return (tr * 128 + 1023) / 1024 * 1024 < 10240 ? 10240 : (tr * 128 + 1023) / 1024 * 1024;
}

struct FusedArgs {
  const uint32_t* masked;  // [1]
  int active;              // score only the active sub-block (scored_bits)
  int H, V;
  float tau;
  int S;
  int32_t* tokens;
  uint32_t* unmask;
  float* pmax_out;
  int32_t* argmax_out;
  float* pm;  // partials [32 positions][part_stride]
  float* ps;
  int32_t* pa;
  int part_stride;    // >= gridDim.x, a multiple of 4
  int tile_rows;      // TR: W rows per vocab tile (the W tensor map's box)
  int32_t* status;    // 0 between calls; a bounded wait that gave up sets it
  uint32_t* arrivals; // 0 between calls
  int32_t* tile_ctr;  // 0 between calls
};

__global__ void __launch_bounds__(kThreads, 1)
    select_fused_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_h,
                        const __grid_constant__ CUtensorMap tm_hp, FusedArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[kMaxStages], empty_bar[kMaxStages];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2];
  __shared__ uint64_t tile_bar[kSlots], tile_free[kSlots];
  __shared__ int tile_q[kSlots];
  __shared__ uint32_t tmem_slot;
  __shared__ float red_m[4][64], red_s[4][64];
  __shared__ int red_a[4][64];
  __shared__ float xpose[4][32 * 33];
  __shared__ float sp[kBlock];
  __shared__ int stok[kBlock];
  __shared__ int pos_of[kBlock];  // position of the r-th masked bit
  __shared__ int s_last;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_k = (a.H + kKStage - 1) / kKStage;
  const int R = gridDim.x;
  const int TR = a.tile_rows;
  const int n_tiles = (a.V + TR - 1) / TR;
  const int w_region = stage_w_bytes(TR);
  const int stage_bytes = w_region + kBBytes;
  int n_stages = kSmemBytes / stage_bytes;
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
    for (int i = 0; i < kSlots; ++i) {
      tc::mbar_init(&tile_bar[i], 1);
      tc::mbar_init(&tile_free[i], 5);  // the MMA issuer and the 4 epilogue warps
    }
    tc::fence_barrier_init();
  }
  // Operand rows 33..47 are never loaded: zero them once in every stage.
  for (int x = threadIdx.x; x < n_stages * (kN - kHpRow - 1) * 8; x += kThreads) {
    const int s = x / ((kN - kHpRow - 1) * 8), rem = x % ((kN - kHpRow - 1) * 8);
    const int row = kHpRow + 1 + rem / 8, c = rem % 8;
    tc::st_shared_v4(tc::smem_u32(smem + s * stage_bytes + w_region + row * 128 + c * 16), 0u, 0u,
                     0u, 0u);
  }
  tc::fence_proxy_async();
  if (warp == 1) tc::tmem_alloc(&tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  griddep_wait();  // first kernel of the call: the caller's inputs are complete after this
  griddep_launch_dependents();
  const uint32_t bits = scored_bits(a.masked[0], a.S, a.active);

  if (warp == 0) {
    // ---------------------------------------------------------- TMA producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_w);
      tc::prefetch_tmap(&tm_h);
      tc::prefetch_tmap(&tm_hp);
      const uint64_t pol_w = tc::policy_evict_first();
      const uint64_t pol_h = tc::policy_evict_last();
      int next = bits ? blockIdx.x : n_tiles;  // the first tile needs no counter
      int s = 0;
      uint32_t ph = 0;
      for (int it = 0;; ++it) {
        const int t = next < n_tiles ? next : -1;
        const int slot = it % kSlots;
        if (!tc::mbar_wait(&tile_free[slot], ((it / kSlots) & 1) ^ 1, a.status)) break;
        tile_q[slot] = t;
        tc::mbar_arrive(&tile_bar[slot]);  // release: consumers read tile_q after their wait
        if (t < 0) break;
        next = R + atomicAdd(a.tile_ctr, 1);  // the next tile, fetched while this one streams
        const int vt = t * TR;  // rows past V (last tile) arrive as zeros
        bool ok = true;
        for (int kb = 0; kb < n_k; ++kb) {
          if (!tc::mbar_wait(&empty_bar[s], ph ^ 1, a.status)) { ok = false; break; }
          uint8_t* st = smem + static_cast<size_t>(s) * stage_bytes;
          uint64_t* bar = &full_bar[s];
          // TR rows of W, 16 + 16 rows of h and the one row of h_prev
          tc::mbar_arrive_expect_tx(bar, (TR + 2 * 16 + 1) * 128);
          tc::tma_load_2d(st, &tm_w, bar, kb * kKStage, vt, pol_w);
          tc::tma_load_2d(st + w_region, &tm_h, bar, kb * kKStage, 0, pol_h);
          tc::tma_load_2d(st + w_region + 16 * 128, &tm_h, bar, kb * kKStage, 16, pol_h);
          tc::tma_load_2d(st + w_region + kHpRow * 128, &tm_hp, bar, kb * kKStage, 0, pol_h);
          if (++s == n_stages) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(kVTile, kN);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int slot = it % kSlots;
        if (!tc::mbar_wait(&tile_bar[slot], (it / kSlots) & 1, a.status)) break;
        const int t = tile_q[slot];
        tc::mbar_arrive(&tile_free[slot]);
        if (t < 0) break;
        const int b = it & 1;
        if (!tc::mbar_wait(&tempty_bar[b], ((it >> 1) & 1) ^ 1, a.status)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + b * 64;
        for (int kb = 0; kb < n_k; ++kb) {
          if (!tc::mbar_wait(&full_bar[s], ph, a.status)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sa = tc::smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
          const uint32_t sb = sa + w_region;
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
    lmh::Run run0 = lmh::run_empty(), run1 = lmh::run_empty();
    for (int it = 0;; ++it) {
      const int slot = it % kSlots;
      if (!tc::mbar_wait_warp(&tile_bar[slot], (it / kSlots) & 1, a.status)) break;
      const int t = tile_q[slot];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tile_free[slot]);
      if (t < 0) break;
      const int b = it & 1;
      if (!tc::mbar_wait_warp(&tfull_bar[b], (it >> 1) & 1, a.status)) break;
      tc::tc_fence_after();
      const int vbase = t * TR + q * 32, vend = min(a.V, t * TR + TR);
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + b * 64;
      lmh::fold_chunk(taddr, xpose[q], lane, vbase, vend, run0);       // h[0..31]
      lmh::fold_chunk(taddr + 32, xpose[q], lane, vbase, vend, run1);  // h_prev, unused
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty_bar[b]);
    }
    red_m[q][lane] = run0.m;
    red_s[q][lane] = run0.s;
    red_a[q][lane] = run0.a;
    red_m[q][32 + lane] = run1.m;
    red_s[q][32 + lane] = run1.s;
    red_a[q][32 + lane] = run1.a;
    tc::named_bar_sync(1, 128);
    const int col = threadIdx.x - 64;
    const int pos = col == kHpRow ? 0 : col + 1;  // position this column scores
    if ((col < kBlock - 1 || col == kHpRow) && ((bits >> pos) & 1u)) {
      Stat st = stat_empty();
#pragma unroll
      for (int qq = 0; qq < 4; ++qq)
        st = stat_combine(st, Stat{red_m[qq][col], red_s[qq][col], red_a[qq][col]});
      const size_t idx = static_cast<size_t>(pos) * a.part_stride + blockIdx.x;
      a.pm[idx] = st.m;
      a.ps[idx] = st.s;
      a.pa[idx] = st.a;
      __threadfence();
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);

  // ------------------------------------------- last CTA: merge and select
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.arrivals, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // Eight lanes per masked position, each reducing its share of the
  // position's partials straight from L2 (all its loads in flight at once):
  // the max and the lowest index attaining it first, then the sum of
  // exp(m_k - max) s_k, one exponential per part.
  const int P = gridDim.x, PS = a.part_stride;
  const int M = __popc(bits);
  if (warp == 0 && ((bits >> lane) & 1u)) pos_of[__popc(bits & ((1u << lane) - 1u))] = lane;
  __syncthreads();
  constexpr int kVecPerLane = 5;  // 8 lanes x 5 x 4 parts >= part_stride (host-checked)
  for (int r0 = warp * 4; r0 < M; r0 += kThreads / 8) {
    const int r = r0 + lane / 8, j = lane % 8;
    const bool live = r < M;
    const size_t row = static_cast<size_t>(live ? pos_of[r] : 0) * PS;
    float4 vm[kVecPerLane], vs[kVecPerLane];
    int4 va[kVecPerLane];
#pragma unroll
    for (int u = 0; u < kVecPerLane; ++u) {
      const int c = j + 8 * u;  // uint4 index within the row
      vm[u] = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (live && 4 * c < PS) {
        vm[u] = __ldcg(reinterpret_cast<const float4*>(a.pm + row) + c);
        vs[u] = __ldcg(reinterpret_cast<const float4*>(a.ps + row) + c);
        va[u] = __ldcg(reinterpret_cast<const int4*>(a.pa + row) + c);
      }
    }
    float mx = -INFINITY;
    int am = 0x7fffffff;
    auto take = [&](float m, int ai, int k) {
      if (k < P && (m > mx || (m == mx && ai < am))) {
        mx = m;
        am = ai;
      }
    };
#pragma unroll
    for (int u = 0; u < kVecPerLane; ++u) {
      const int k = 4 * (j + 8 * u);
      take(vm[u].x, va[u].x, k);
      take(vm[u].y, va[u].y, k + 1);
      take(vm[u].z, va[u].z, k + 2);
      take(vm[u].w, va[u].w, k + 3);
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, mx, o);
      const int oa = __shfl_xor_sync(0xffffffffu, am, o);
      if (om > mx || (om == mx && oa < am)) {
        mx = om;
        am = oa;
      }
    }
    float sum = 0.f;
    auto add = [&](float m, float sv, int k) {
      if (k < P && m != -INFINITY) sum += sv * expf(m - mx);
    };
#pragma unroll
    for (int u = 0; u < kVecPerLane; ++u) {
      const int k = 4 * (j + 8 * u);
      add(vm[u].x, vs[u].x, k);
      add(vm[u].y, vs[u].y, k + 1);
      add(vm[u].z, vs[u].z, k + 2);
      add(vm[u].w, vs[u].w, k + 3);
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (live && j == 0) {
      sp[r] = sum > 0.f ? 1.f / sum : 0.f;  // p_max = exp(max - max) / sum
      stok[r] = am;
    }
  }
  __syncthreads();
  if (warp == 0) {
    const bool is_m = (bits >> lane) & 1u;
    const int r = __popc(bits & ((1u << lane) - 1u));
    if (__ldcg(a.status) != 0)
      no_decision_sequence(0, a.unmask, a.pmax_out, a.argmax_out);
    else
      select_sequence(0, bits, is_m ? sp[r] : 0.f, is_m ? stok[r] : -1, a.tau, a.S, a.tokens,
                      a.unmask, a.pmax_out, a.argmax_out);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // ready for the next call on this workspace
    *a.arrivals = 0u;
    *a.tile_ctr = 0;
    *a.status = 0;
  }
}

}  // namespace

bool select_fused_supported(int dtype, int batch, int hidden) {
  return dtype == BD_BF16 && batch == 1 && hidden % 8 == 0 &&
         select_fused_part_stride() <= 8 * 5 * 4;  // the merge's 8 lanes x 5 x float4
}

int select_fused_part_stride() { return (lmh::sm_count() + 3) / 4 * 4; }

cudaError_t launch_select_fused(int hidden, int vocab, const void* h, const void* h_prev,
                                const void* w, const uint32_t* masked, float tau, int sub_block,
                                int32_t* tokens, uint32_t* unmask, float* pmax_out,
                                int32_t* argmax_out, float* pm, float* ps, int32_t* pa,
                                int32_t* header, int active, cudaStream_t st) {
  // Tile rows: the fewest rounds of one tile per CTA that cover the
  // vocabulary with tiles of at most 128 rows, then the smallest tile size
  // for that many tiles (at least kMinTileRows).
  const int R = lmh::sm_count();
  const long long rounds = (static_cast<long long>(vocab) + static_cast<long long>(R) * kVTile - 1) /
                           (static_cast<long long>(R) * kVTile);
  int tr = static_cast<int>((vocab + rounds * R - 1) / (rounds * R));
  tr = tr < kMinTileRows ? kMinTileRows : (tr > kVTile ? kVTile : tr);
  CUtensorMap tm_w, tm_h, tm_hp;
  if (!lmh::make_tmap_2d(&tm_w, w, static_cast<uint64_t>(vocab), static_cast<uint64_t>(hidden),
                         static_cast<uint32_t>(tr)) ||
      !lmh::make_tmap_2d(&tm_h, h, kBlock, static_cast<uint64_t>(hidden), 16) ||
      !lmh::make_tmap_2d(&tm_hp, h_prev, 1, static_cast<uint64_t>(hidden), 1))
    return cudaErrorInvalidValue;
  FusedArgs a{};
  a.masked = masked;
  a.active = active;
  a.H = hidden;
  a.V = vocab;
  a.tau = tau;
  a.S = sub_block;
  a.tokens = tokens;
  a.unmask = unmask;
  a.pmax_out = pmax_out;
  a.argmax_out = argmax_out;
  a.pm = pm;
  a.ps = ps;
  a.pa = pa;
  a.part_stride = select_fused_part_stride();
  a.tile_rows = tr;
  a.status = header + 1;
  a.arrivals = reinterpret_cast<uint32_t*>(header + 2);
  a.tile_ctr = header + 3;
  cudaFuncSetAttribute(select_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kSmemBytes + 1024);
  const cudaError_t e = launch_pdl(select_fused_kernel, dim3(lmh::sm_count()), dim3(kThreads),
                                   kSmemBytes + 1024, st, tm_w, tm_h, tm_hp, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd
