// bd_block_attn on the 5th-generation tensor cores (bf16 storage, head_dim
// 128): the current 32-token block attends to [cached pages ; itself]
// ("Fast-dLLM v2: Efficient Block-Diffusion LLM", overall framework and key
// design 3 -- block-internal bidirectional, block-causal across blocks, the
// finished blocks read from the block-level KV cache).
//
// CTA = (split-KV chunk, KV head g, sequence s).  Its query rows are the
// G = Hq/Hkv heads of group g times the block's 32 positions (row r = head
// (r / 32) of the group, position r % 32), one or two 128-row tiles Q_t,
// loaded once by TMA into shared memory.  The chunk's pages stream in
// 128-key steps (four pages, TMA, 128-byte swizzle) through a ring of four
// 32 KB slots holding K_0, V_0, K_1, V_1, K_2, ... in turn: K_j's slot is
// released as soon as S(j) = Q K_j^T has been computed, V_j's after P V_j,
// so the loads of step j+2 start about two steps before they are needed.
//
// Tensor memory (512 columns): S_t at 128 t (fp32; P_t is written over its
// first 64 columns as packed bf16), O_t at 256 + 128 t (fp32).
//
//   warp 1 (one thread)  ping-pong over the query tiles, per stage j:
//                        O_t += P_t(j) V_j (TS MMA, P from TMEM), then
//                        S_t(j+1) = Q_t K_{j+1}^T (SS MMA, N = 128 keys).
//                        MMAs of one thread execute in issue order, so
//                        S_t(j+1) overwrites P_t(j) only after P V has read
//                        it, and while tile t's softmax works the tensor core
//                        runs the other tile's products.
//   warps 4+4t .. 7+4t   one thread per query row: online softmax in base 2
//                        (scores scaled by log2(e)/sqrt(d) inside one FMA),
//                        P as bf16 over S_t, lazy rescale of its O row when
//                        the running max grows by more than 2^8.  Tile t's
//                        tensor-memory stores happen only when none of tile
//                        t's own products is in flight.
//   warp 0               TMA producer: Q, then the K/V pages (16 lanes issue
//                        the 16 boxes of a stage).
//
// The chunk's (m, l, O) go to the workspace for attn_merge_kernel, or --
// when one chunk covers the whole sequence -- O / l straight to the output.
#include <cstring>

#include "bd_common.cuh"
#include "tc_common.cuh"

namespace bd {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 384;               // 12 warps
constexpr int kKeys = 128;                   // keys per step (four pages)
constexpr int kSlots = 4;                    // ring slots of one K or V step each
constexpr int kPreSteps = kSlots / 2;        // steps whose slots are free at the start
constexpr int kQTileBytes = 128 * kD * 2;    // 32 KB
constexpr int kKVBytes = kKeys * kD * 2;     // 32 KB each for K and V
constexpr int kMaxChunkPages = 1024;
constexpr float kRescaleThreshold = 8.f;     // log2 units
// pairs of scores whose exponentials are evaluated on the FMA pipe: one in
// four (a third or a half measured slower: the polynomial's issue cost then
// outweighs the MUFU time it saves)
__device__ __forceinline__ constexpr bool kPolyPair(int k) { return (k & 3) == 3; }
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr int kOffQ = 0;
constexpr int kOffKV = 2 * kQTileBytes;
constexpr int kSmemBytes = kOffKV + kSlots * kKVBytes + 1024;  // + alignment slack

struct AttnTcArgs {
  const int32_t* page_table;
  const int32_t* n_blocks;
  int max_blocks;
  long long n_pages;
  int Hq, Hkv, G, R;       // R = G * 32 query rows per CTA
  int ppc, max_chunks;
  int kv_rows_total;       // rows of the page-pool tensor map (OOB row for padding)
  float* part_o;
  float* part_ml;
  bf16* out;
  int32_t* status;
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                   const __grid_constant__ CUtensorMap tm_blk,
                   const __grid_constant__ CUtensorMap tm_out,
                   const __grid_constant__ CUtensorMap tm_po, AttnTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t q_full;
  __shared__ uint64_t kv_full[kSlots], kv_empty[kSlots];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int pages[kMaxChunkPages];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int c = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
  const int nb = min(max(a.n_blocks[s], 0), a.max_blocks);
  const int total = nb + 1;  // cached pages + the current block
  const int p0 = c * a.ppc;
  if (p0 >= total) {
    griddep_wait();  // completes only after the prep kernel
    return;
  }
  const int p1 = min(total, p0 + a.ppc);
  const int n_pg = p1 - p0;
  const int n_tiles = (n_pg + 3) / 4;
  const int nq = (a.R + 127) / 128;

  for (int i = threadIdx.x; i < n_pg; i += blockDim.x) {
    const int p = p0 + i;
    int pg = -1;  // -1: the current block's page in the workspace
    if (p < nb) {
      pg = a.page_table[static_cast<size_t>(s) * a.max_blocks + p];
      BD_CHECK(pg >= 0 && pg < a.n_pages, kCheckPageId, pg);
      if (pg < 0 || pg >= a.n_pages) pg = -2;  // host-validated; read zeros if not
    }
    pages[i] = pg;
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    for (int i = 0; i < kSlots; ++i) {
      tc::mbar_init(&kv_full[i], 1);
      tc::mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      tc::mbar_init(&s_full[t], 1);
      tc::mbar_init(&p_full[t], 4);
      tc::mbar_init(&pv_done[t], 1);
    }
    tc::fence_barrier_init();
    tc::fence_proxy_async();
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t sbase = tc::smem_u32(smem);
  griddep_launch_dependents();
  if (warp != 0) griddep_wait();  // outputs are written after the prep kernel completes

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    // The whole warp: lane 0 arms the stage's barrier, then lanes 0..15 each
    // issue one of its sixteen 4 KB boxes (page, K or V, d half).
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_kv);
      tc::prefetch_tmap(&tm_blk);
    }
    const uint64_t pol_kv = tc::policy_evict_first();
    const uint64_t pol_q = tc::policy_evict_last();
    // Cached pages were committed before this call, so the first stages of
    // cache pages load while the prep kernel still runs; Q and the current
    // block's page (both written by prep) load after the grid dependency.
    bool dep = false;
    auto wait_prep_load_q = [&]() {
      griddep_wait();
      dep = true;
      if (lane == 0) {
        const int qrow0 = (s * a.Hq + g * a.G) * kBlock;
        tc::mbar_arrive_expect_tx(&q_full, nq * kQTileBytes);
        for (int t = 0; t < nq; ++t)
          for (int dh = 0; dh < 2; ++dh)
            tc::tma_load_2d(smem + kOffQ + t * kQTileBytes + dh * (kQTileBytes / 2), &tm_q,
                            &q_full, dh * 64, qrow0 + 128 * t, pol_q);
      }
      __syncwarp();
    };
    const bool has_blk = p1 == total;  // the chunk ends with the current block's page
    const int pg = (lane >> 1) & 3, dh = lane & 1;
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      if (!dep && (j >= kPreSteps || (has_blk && j == n_tiles - 1))) wait_prep_load_q();
      for (int kv = 0; kv < 2; ++kv) {  // K_j, then V_j: ring buffer b = 2 j + kv
        const int b = 2 * j + kv, sl = b % kSlots;
        if (!tc::mbar_wait_warp(&kv_empty[sl], ((b / kSlots) & 1) ^ 1, a.status)) {
          ok = false;
          break;
        }
        if (lane == 0) tc::mbar_arrive_expect_tx(&kv_full[sl], kKVBytes);
        __syncwarp();
        if (lane < 8) {  // the step's 8 boxes: 4 pages x 2 halves of d
          const int i = 4 * j + pg;
          const CUtensorMap* m = &tm_kv;
          int row;
          if (i >= n_pg || pages[i] == -2) {  // padding page: rows past the end read as zeros
            row = a.kv_rows_total;
          } else if (pages[i] == -1) {
            m = &tm_blk;
            row = ((s * 2 + kv) * a.Hkv + g) * kBlock;
          } else {
            row = ((pages[i] * 2 + kv) * a.Hkv + g) * kBlock;
          }
          tc::tma_load_2d(smem + kOffKV + sl * kKVBytes + dh * (kKVBytes / 2) + pg * 4096, m,
                          &kv_full[sl], dh * 64, row, pol_kv);
        }
        __syncwarp();
      }
    }
    // Fewer steps than kPreSteps, none holding the current block (the loop
    // cannot stop early before `dep`: the first kPreSteps steps' slots are
    // free).
    if (!dep) wait_prep_load_q();
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = tc::idesc_bf16_f32(128, kKeys);
      const uint32_t id_pv = tc::idesc_bf16_f32_bmn(128, kD);
      auto full = [&](int b) { return tc::mbar_wait(&kv_full[b % kSlots], (b / kSlots) & 1, a.status); };
      // Shared-memory descriptors built once; a stage, a query tile or a
      // K-step only moves the start-address field (bits [0,14), 16-byte
      // units), so each MMA costs two 64-bit adds.  The issuing thread shares
      // its SM sub-partition with softmax warps, so every instruction it
      // saves keeps the tensor core fed.
      const uint64_t qdesc0 = tc::sdesc_kmajor_sw128(sbase + kOffQ);
      const uint64_t kdesc0 = tc::sdesc_kmajor_sw128(sbase + kOffKV);
      const uint64_t vdesc0 = tc::sdesc_mnmajor_sw128(sbase + kOffKV, kKVBytes / 2);
      constexpr uint64_t kSlotStep = kKVBytes >> 4, kQStep = kQTileBytes >> 4;
      constexpr uint64_t kHalfStep = (kKVBytes / 2) >> 4;  // the second 64 of d (Q and K alike)
      static_assert(kQTileBytes / 2 == kKVBytes / 2, "Q and K tiles split d at the same offset");
      auto issue_qk = [&](int t, int j) {  // S_t = Q_t K_j^T, K = d: 8 steps of 16
        const uint64_t qd = qdesc0 + static_cast<uint64_t>(t) * kQStep;
        const uint64_t kd = kdesc0 + static_cast<uint64_t>((2 * j) % kSlots) * kSlotStep;
        const uint32_t d = tmem + kColS + t * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t o = (kk >> 2) * kHalfStep + (kk & 3) * 2;  // + 32 bytes per K-step
          tc::mma_bf16_ss(d, qd + o, kd + o, id_qk, kk != 0);
        }
        tc::mma_commit(&s_full[t]);
      };
      bool ok = tc::mbar_wait(&q_full, 0, a.status) && full(0);
      tc::tc_fence_after();
      for (int t = 0; t < nq && ok; ++t) issue_qk(t, 0);
      if (ok) tc::mma_commit(&kv_empty[0]);  // K_0 has been read once its products are done
      for (int j = 0; j < n_tiles && ok; ++j) {
        const bool more = j + 1 < n_tiles;
        const uint64_t vd = vdesc0 + static_cast<uint64_t>((2 * j + 1) % kSlots) * kSlotStep;
        for (int t = 0; t < nq && ok; ++t) {
          if (!tc::mbar_wait(&p_full[t], j & 1, a.status)) { ok = false; break; }
          if (t == 0 && !full(2 * j + 1)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t dO = tmem + kColO + t * 128, aP = tmem + kColS + t * 128;
#pragma unroll
          for (int kk = 0; kk < kKeys / 16; ++kk)  // O_t += P_t V_j, K = keys: 8 steps of 16
            tc::mma_bf16_ts(dO, aP + kk * 8, vd + kk * ((16 * 128) >> 4), id_pv, (j | kk) != 0);
          tc::mma_commit(&pv_done[t]);
          if (t == nq - 1) tc::mma_commit(&kv_empty[(2 * j + 1) % kSlots]);  // V_j read
          if (more) {
            if (t == 0 && !full(2 * j + 2)) { ok = false; break; }
            tc::tc_fence_after();
            issue_qk(t, j + 1);
          }
        }
        if (ok && more) tc::mma_commit(&kv_empty[(2 * j + 2) % kSlots]);  // K_{j+1} read
      }
    }
  } else if (warp >= 4 && (warp - 4) / 4 < nq) {
    // ------------------------------------------------ softmax / correction
    const int t = (warp - 4) / 4;
    const int q = warp & 3;
    const int r = 128 * t + 32 * q + lane;  // query row of this thread
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const float scale = kLog2e * rsqrtf(static_cast<float>(kD));
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    const uint32_t sbuf = tmem + lane_off + kColS + t * 128;
    // A warp whose 32 rows are all padding of the last query tile (G * 32 not
    // a multiple of 128) only keeps the barrier protocol: its P rows are never
    // written, so P V gives garbage in output rows that are never stored.
    const bool pad_warp = 32 * (r / 32) >= a.R;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int valid = min(kKeys, kBlock * (n_pg - 4 * j));
      // S_t(j) complete also means tile t's earlier products (P V of stage
      // j-1 included) have completed: none of tile t's MMAs is in flight.
      if (!tc::mbar_wait_warp(&s_full[t], j & 1, a.status)) { ok = false; break; }
      tc::tc_fence_after();
      if (pad_warp) {
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&p_full[t]);
        continue;
      }
      uint32_t sr[128];
      float alpha = 1.f;
      bool rescale = false;
      float2 rk[2];
      int jmax;
      // The 16 pairs of 32-column chunk cc: p = 2^(s * scale - m) in paired
      // fp32 arithmetic, a quarter of the pairs on the FMA pipe, the rest on
      // MUFU; packed in place, sr[k] <- (p_2k, p_2k+1).
      auto exps = [&](int cc) {
        const float2 sc2 = make_float2(scale, scale), nm2 = make_float2(-m, -m);
#pragma unroll
        for (int k = 16 * cc; k < 16 * cc + 16; ++k) {
          const float2 x = ffma2(make_float2(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])),
                                 sc2, nm2);
          const float2 e = kPolyPair(k) ? poly_exp2x2(x, jmax) : make_float2(fast_exp2(x.x), fast_exp2(x.y));
          rk[k & 1] = fadd2(rk[k & 1], e);
          sr[k] = tc::pack_bf16x2(e.x, e.y);
        }
      };
      // A full stage after the first: the exponentials are taken against the
      // running max m as it stands, without a max pass, and each 32-column
      // TMEM load of S overlaps the exponentials of the chunk before.  That
      // equals the max-pass result whenever no score of the stage exceeds m
      // by more than kRescaleThreshold (the only case in which the max pass
      // moves m): a stage sum of exponentials <= 2^8 and a largest integer
      // part <= 8 among the polynomial pairs prove it.  Otherwise, and at the
      // first or a partial stage, the max pass runs and the exponentials are
      // taken again (S is still in TMEM).
      bool done = false;
      if (j > 0 && valid == kKeys) {  // warp-uniform
        rk[0] = rk[1] = make_float2(0.f, 0.f);
        jmax = 0;
        tc::tmem_ld_32x32b_x32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          tc::tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
          if (cc < 3)
            tc::tmem_ld_32x32b_x32(sbuf + (cc + 1) * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * (cc + 1)]));
          exps(cc);
        }
        const float sum = (rk[0].x + rk[0].y) + (rk[1].x + rk[1].y);
        static_assert(kRescaleThreshold == 8.f, "the bounds below are 2^8 and 8");
        done = !__any_sync(0xffffffffu, !(sum <= 256.f) || jmax > 8);
      }
      if (!done) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          tc::tmem_ld_32x32b_x32(sbuf + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
        tc::tmem_ld_wait();
        if (valid < kKeys) {  // warp-uniform: only the last stage of a chunk can be partial
#pragma unroll
          for (int k = 32; k < 128; ++k)
            if (k >= valid) sr[k] = __float_as_uint(-INFINITY);
        }
        float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int k = 0; k < 128; k += 2)
          mk[(k >> 1) & 3] = tc::fmax3(mk[(k >> 1) & 3], __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
        const float mt = fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])) * scale;
        const float m_new = fmaxf(m, mt);
        rescale = (m == -INFINITY) || (m_new - m > kRescaleThreshold);
        if (rescale) {
          alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
          m = m_new;
        }
        rk[0] = rk[1] = make_float2(0.f, 0.f);
        jmax = 0;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) exps(cc);
      }
      l = l * alpha + ((rk[0].x + rk[0].y) + (rk[1].x + rk[1].y));
      // TMEM accesses are warp-collective, so the warp rescales together when
      // any of its rows needs it, the other rows with a factor of 1.
      const bool need = rescale && j > 0;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? alpha : 1.f;
        const uint32_t o_addr = tmem + lane_off + kColO + t * 128;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tc::tmem_ld_32x32b_x32(o_addr + cc * 32, ov);
          tc::tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * f);
          tc::tmem_st_32x32b_x32(o_addr + cc * 32, ov);
        }
      }
      // P_t(j) over the first 64 columns of S_t
      tc::tmem_st_32x32b_x32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tc::tmem_st_32x32b_x32(sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------------- output
    // Warp-uniform: the wait verdict is shared by the warp, and R is a
    // multiple of 32, so each warp's rows are all valid or all padding.
    if (ok && tc::mbar_wait_warp(&pv_done[t], (n_tiles - 1) & 1, a.status)) {
      tc::tc_fence_after();
      if (32 * (r / 32) < a.R) {
        // The warp's 32 rows are the 32 positions of one query head h.  O
        // goes out by TMA tile stores from the warp's 8 KB slice of its
        // query tile's Q buffer (free once the tile's last product is done),
        // written in the store's 128-byte-swizzled layout: bf16 O / l as two
        // (64 d x 32 positions) boxes of `out`, or the fp32 chunk partial as
        // four (32 d x 32 positions) boxes of the partial buffer.
        const int h = g * a.G + r / kBlock;
        const int pos = r % kBlock;
        const bool single = (total <= a.ppc) || (a.max_chunks == 1);
        const uint32_t o_addr = tmem + lane_off + kColO + t * 128;
        const float inv = 1.f / l;
        const size_t prow0 = ((static_cast<size_t>(s) * a.Hq + h) * a.max_chunks + c) * kBlock;
        const size_t prow_idx = prow0 + pos;
        uint8_t* stg = smem + kOffQ + t * kQTileBytes + q * 8192;
        if (single) {
#pragma unroll 1
          for (int dh = 0; dh < 2; ++dh) {  // 64 d per box
            uint8_t* box = stg + dh * 4096;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t ov[32];
              tc::tmem_ld_32x32b_x32(o_addr + dh * 64 + half * 32, ov);
              tc::tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 4; ++k) {  // 8 bf16 = one 16-byte chunk
                uint4 v;
                v.x = tc::pack_bf16x2(__uint_as_float(ov[8 * k + 0]) * inv, __uint_as_float(ov[8 * k + 1]) * inv);
                v.y = tc::pack_bf16x2(__uint_as_float(ov[8 * k + 2]) * inv, __uint_as_float(ov[8 * k + 3]) * inv);
                v.z = tc::pack_bf16x2(__uint_as_float(ov[8 * k + 4]) * inv, __uint_as_float(ov[8 * k + 5]) * inv);
                v.w = tc::pack_bf16x2(__uint_as_float(ov[8 * k + 6]) * inv, __uint_as_float(ov[8 * k + 7]) * inv);
                const int chunk = half * 4 + k;
                *reinterpret_cast<uint4*>(box + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = v;
              }
            }
          }
          tc::fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tc::tma_store_3d(&tm_out, stg, 0, h, s * kBlock);
            tc::tma_store_3d(&tm_out, stg + 4096, 64, h, s * kBlock);
            tc::bulk_commit();
            tc::bulk_wait_read<0>();
          }
          __syncwarp();
        } else {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {  // 32 fp32 per box
            uint8_t* box = stg + (cc & 1) * 4096;
            if (cc >= 2) {  // the box's previous store must have read it
              if (lane == 0) tc::bulk_wait_read<1>();
              __syncwarp();
            }
            uint32_t ov[32];
            tc::tmem_ld_32x32b_x32(o_addr + cc * 32, ov);
            tc::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 8; ++k)
              *reinterpret_cast<uint4*>(box + lane * 128 + ((k ^ (lane & 7)) << 4)) =
                  make_uint4(ov[4 * k], ov[4 * k + 1], ov[4 * k + 2], ov[4 * k + 3]);
            tc::fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tc::tma_store_2d(&tm_po, box, cc * 32, static_cast<int>(prow0));
              tc::bulk_commit();
            }
          }
          if (lane == 0) tc::bulk_wait_read<0>();
          __syncwarp();
        }
        if (!single) {
          a.part_ml[prow_idx * 2 + 0] = m;
          a.part_ml[prow_idx * 2 + 1] = l;
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), rows};
  const cuuint64_t strides[1] = {kD * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output [rows][heads][128] bf16 viewed as (d, head, row): box = 32 rows of
// one head, 64 d wide, 128-byte swizzle (tile stores).
bool make_tmap_out(CUtensorMap* m, const void* base, uint64_t rows, uint32_t heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), heads, rows};
  const cuuint64_t strides[2] = {kD * 2, static_cast<cuuint64_t>(heads) * kD * 2};
  const cuuint32_t box[3] = {64, 1, kBlock};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 partial O [rows][128]: box = 32 rows x 32 floats (128 bytes), 128-byte swizzle.
bool make_tmap_part(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), rows};
  const cuuint64_t strides[1] = {kD * 4};
  const cuuint32_t box[2] = {32, kBlock};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_tc_supported(const bd_attn_shape& sh) {
  const int G = sh.n_heads_q / sh.n_heads_kv;
  return sh.dtype == BD_BF16 && sh.head_dim == kD && G * kBlock <= 256;
}

int attn_tc_max_chunk_pages() { return kMaxChunkPages; }

cudaError_t launch_attn_tc(const bd_attn_shape& sh, const bd_kv_cache& c, int ppc, int max_chunks,
                           const void* ws_q, const void* ws_blk, float* part_o, float* part_ml,
                           void* out, int32_t* status, cudaStream_t st) {
  const int B = c.batch, Hq = sh.n_heads_q, Hkv = sh.n_heads_kv;
  CUtensorMap tm_q, tm_kv, tm_blk, tm_out, tm_po;
  const uint64_t kv_rows = static_cast<uint64_t>(c.n_pages) * 2 * Hkv * kBlock;
  if (kv_rows >= (1ull << 31)) return cudaErrorInvalidValue;
  if (!make_tmap(&tm_q, ws_q, static_cast<uint64_t>(B) * Hq * kBlock, 128) ||
      !make_tmap(&tm_kv, c.pages, kv_rows, kBlock) ||
      !make_tmap(&tm_blk, ws_blk, static_cast<uint64_t>(B) * 2 * Hkv * kBlock, kBlock) ||
      !make_tmap_out(&tm_out, out, static_cast<uint64_t>(B) * kBlock, Hq))
    return cudaErrorInvalidValue;
  std::memset(&tm_po, 0, sizeof(tm_po));  // unused unless a sequence spans several chunks
  if (max_chunks > 1 &&
      !make_tmap_part(&tm_po, part_o, static_cast<uint64_t>(B) * Hq * max_chunks * kBlock))
    return cudaErrorInvalidValue;
  AttnTcArgs a{};
  a.page_table = c.page_table;
  a.n_blocks = c.n_blocks;
  a.max_blocks = c.max_blocks;
  a.n_pages = c.n_pages;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.R = a.G * kBlock;
  a.ppc = ppc;
  a.max_chunks = max_chunks;
  a.kv_rows_total = static_cast<int>(kv_rows);
  a.part_o = part_o;
  a.part_ml = part_ml;
  a.out = static_cast<bf16*>(out);
  a.status = status;
  cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  const cudaError_t e = launch_pdl(attn_tc_kernel, dim3(max_chunks, Hkv, B), dim3(kThreads),
                                   kSmemBytes, st, tm_q, tm_kv, tm_blk, tm_out, tm_po, a);
  if (e != cudaSuccess) return e;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd

#ifdef BD_DEVICE_CHECKS
namespace bd {
cudaError_t check_word_attn_tc(int* host2, bool reset) { return read_check_word(host2, reset); }
}  // namespace bd
#endif
