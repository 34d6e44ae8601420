// bd_block_mask_attn on the 5th-generation tensor cores (bf16, head_dim 128):
// attention of the training forward over [noisy x_t ; clean x_0] under the
// block-diffusion mixed mask ("Fast-dLLM v2: Efficient Block-Diffusion
// LLM", key design 2).  With blk(i) = (i mod L) / D a noisy query sees the
// noisy keys of its own block and the clean keys of earlier blocks; a clean
// query sees the clean keys of its own and earlier blocks.
//
// Work item = (128-row query tile, pair of query heads of one KV group,
// view); one persistent CTA per SM works through its share of the items, so
// the next item's query tiles and first K/V tile load while the current one
// finishes.  The two heads are the item's two query tiles Q_0, Q_1 (TMA,
// shared memory); they read the same K/V.  Of the 2L/128 key tiles only
// those the mask leaves visible to the query tile are streamed (two 128-key
// K/V stages); a tile that is only partly visible is masked in the softmax.
// Per key tile the MMA thread ping-pongs O_t += P_t V (TS MMA, P in TMEM) and
// S_t = Q_t K^T (SS MMA); one thread per query row runs the base-2 online
// softmax with lazy rescaling, as in attn_tc.cu.  Every key of a row is
// seen within one item, so O / l goes straight to the output.
//
// Views that share a sample: the two complementary-mask views of one
// training sample differ only in their noisy stream; the clean stream x_0,
// and with it every clean query's output (clean queries see clean keys
// only), is the same.  With views > 1 the clean query tiles of a sample are
// computed once and stored into the rows of each of its views.
#include "bd_common.cuh"
#include "mask_attn.cuh"
#include "tc_common.cuh"

namespace bd {
namespace {

constexpr int kD = 128;
constexpr int kThreads = 384;
constexpr int kT = 128;                     // query rows per tile = keys per stage
constexpr int kStages = 2;
constexpr int kQTileBytes = kT * kD * 2;    // 32 KB
constexpr int kKVBytes = kT * kD * 2;       // 32 KB each for K and V
constexpr float kRescaleThreshold = 8.f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;
constexpr int kOffQ = 0;
constexpr int kOffKV = 2 * kQTileBytes;
constexpr int kOffStg = kOffKV + kStages * 2 * kKVBytes;  // 8 softmax warps x one 4 KB output box
constexpr int kSmemBytes = kOffStg + 8 * 4096 + 1024;      // + alignment slack

struct MaskArgs {
  int L, D, Hq, Hkv, G;
  int n_qt;       // 2L / 128
  int per_group;  // query-head pairs per KV group: ceil(G / 2)
  int n_seqs;     // entries (samples x views)
  int views;      // consecutive entries that share one clean stream
  int n_samples;  // n_seqs / views
  int n_items;    // n_qt / 2 x (n_seqs + n_samples) x per_group x Hkv work items
  bf16* out;
  int32_t* status;
};

// A 128-row tile of the 2L sequence: its stream and block range.
struct Span {
  bool noisy;
  int b_lo, b_hi;
};
__device__ __forceinline__ Span span_of(int tile, int L, int D) {
  const int r0 = tile * kT;
  const bool noisy = r0 < L;
  const int loc = noisy ? r0 : r0 - L;
  return Span{noisy, loc / D, (loc + kT - 1) / D};
}
// 0: no pair visible, 1: some, 2: all (no element mask needed).
__device__ __forceinline__ int tile_visibility(Span q, Span k, int D) {
  if (!q.noisy && k.noisy) return 0;
  if (q.noisy && k.noisy) {
    if (k.b_hi < q.b_lo || k.b_lo > q.b_hi) return 0;
    return (q.b_lo == q.b_hi && k.b_lo == k.b_hi && q.b_lo == k.b_lo) ? 2 : 1;
  }
  if (q.noisy) {  // noisy query, clean key: blk(key) < blk(query)
    if (k.b_lo >= q.b_hi) return 0;
    return k.b_hi < q.b_lo ? 2 : 1;
  }
  if (k.b_lo > q.b_hi) return 0;  // clean query, clean key: blk(key) <= blk(query)
  return k.b_hi <= q.b_lo ? 2 : 1;
}
__device__ __forceinline__ bool pair_visible(int i, int j, int L, int D) {
  const bool qn = i < L, kn = j < L;
  const int bq = (qn ? i : i - L) / D, bk = (kn ? j : j - L) / D;
  if (qn) return kn ? (bk == bq) : (bk < bq);
  return kn ? false : (bk <= bq);
}

// One work item = (128-row query tile, pair of query heads of one KV group,
// entry): the unit the kernel used to give each CTA.  The grid is one
// persistent CTA per SM; CTA c takes items c, then 2G-1-c, then 2G+c, ...
// (G CTAs, a snake over the items ranked heaviest first), so each SM gets
// about the same number of key tiles.  Every role walks the same item
// sequence and finds each item's visible key tiles itself.
struct Item {
  int qt, h0, nq, g, n;
  Span qs;
};
template <bool kViews>
__device__ __forceinline__ Item item_of(int i, const MaskArgs& a) {
  const int pairs = a.per_group * a.Hkv;
  const int half = a.n_qt / 2;
  Item it;
  int pr;
  if constexpr (!kViews) {
    // Heaviest query tiles first: noisy query tile w and clean query tile
    // n_qt / 2 + w both see w + 1 (or w + 2) key tiles, so the ranks take
    // them in pairs from the last w down.
    const int rank = i / (pairs * a.n_seqs), rem = i % (pairs * a.n_seqs);
    const int wq = half - 1 - rank / 2;
    it.n = rem / pairs;
    pr = rem % pairs;
    it.qt = (rank & 1) ? wq : half + wq;
  } else {
    // The same levels, each holding the clean items (one per sample and
    // head pair, on the sample's first view) and then the noisy items (one
    // per entry and head pair).
    const int n_clean = pairs * a.n_samples, per_level = n_clean + pairs * a.n_seqs;
    const int lvl = i / per_level;
    int rem = i - lvl * per_level;
    const int wq = half - 1 - lvl;
    if (rem < n_clean) {
      it.n = (rem / pairs) * a.views;
      pr = rem % pairs;
      it.qt = half + wq;
    } else {
      rem -= n_clean;
      it.n = rem / pairs;
      pr = rem % pairs;
      it.qt = wq;
    }
  }
  it.g = pr / a.per_group;
  const int w = pr % a.per_group;
  it.h0 = it.g * a.G + 2 * w;                 // first head of the pair
  it.nq = (2 * w + 1 < a.G) ? 2 : 1;          // odd G: the last pair has one head
  it.qs = span_of(it.qt, a.L, a.D);
  return it;
}
// The k-th item of CTA c (or -1 past the end of a partial last round).
__device__ __forceinline__ int item_index(int k, int c, int n_ctas, int n_items) {
  const int i = k * n_ctas + ((k & 1) ? n_ctas - 1 - c : c);
  return i < n_items ? i : -1;
}
// The key tiles the mask leaves visible to a query tile, in increasing
// order, form two runs: noisy tiles [a0, a0 + na) (a noisy query: the tiles
// that overlap its own blocks) and clean tiles [n_qt / 2, c1) (the clean
// blocks before a noisy query's blocks, or up to and including a clean
// query's).  Tile j of the item is vis_tile(v, j); there are v.n.
struct VisRanges {
  int a0, na, c1, n;
};
__device__ __forceinline__ VisRanges visible_ranges(const Span& qs, const MaskArgs& a) {
  const int half = a.n_qt / 2;
  VisRanges v;
  if (qs.noisy) {
    v.a0 = qs.b_lo * a.D / kT;
    v.na = min(half, ((qs.b_hi + 1) * a.D + kT - 1) / kT) - v.a0;
    v.c1 = half + min(half, (qs.b_hi * a.D + kT - 1) / kT);
  } else {
    v.a0 = 0;
    v.na = 0;
    v.c1 = half + min(half, ((qs.b_hi + 1) * a.D + kT - 1) / kT);
  }
  v.n = v.na + (v.c1 - half);
  return v;
}
__device__ __forceinline__ int vis_tile(const VisRanges& v, int j, int half) {
  return j < v.na ? v.a0 + j : half + (j - v.na);
}

template <bool kViews>
__global__ void __launch_bounds__(kThreads, 1)
    mask_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_out, MaskArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // q_free: the item's last Q K^T products are done (Q may be replaced);
  // o_free[t]: tile t's O has been read out (the next item may overwrite it)
  __shared__ uint64_t q_full, q_free;
  __shared__ uint64_t kv_full[kStages], kv_empty[kStages];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  __shared__ uint32_t tmem_slot;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int cta = blockIdx.x, n_ctas = gridDim.x;
  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    tc::mbar_init(&q_free, 1);
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&kv_full[i], 1);
      tc::mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      tc::mbar_init(&s_full[t], 1);
      tc::mbar_init(&p_full[t], 4);
      tc::mbar_init(&pv_done[t], 1);
      tc::mbar_init(&o_free[t], 4);
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

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    // Per item: the first visible K/V tile, then (once the previous item's
    // Q K^T products are done) the query tiles, then the remaining tiles.
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
    }
    const uint64_t pol_kv = tc::policy_evict_last();  // K/V tiles are re-read by other items
    int st = 0, kq = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int k = 0; k * n_ctas < a.n_items && ok; ++k) {
      const int i = item_index(k, cta, n_ctas, a.n_items);
      if (i < 0) continue;
      const Item it = item_of<kViews>(i, a);
      const int row_base = it.n * 2 * a.L;
      const VisRanges v = visible_ranges(it.qs, a);
      for (int j = 0; j < v.n; ++j) {
        const int kt = vis_tile(v, j, a.n_qt / 2);
        if (!tc::mbar_wait_warp(&kv_empty[st], ph ^ 1, a.status)) { ok = false; break; }
        if (lane == 0) tc::mbar_arrive_expect_tx(&kv_full[st], 2 * kKVBytes);
        __syncwarp();
        if (lane < 4) {  // lane = (K or V, d half)
          const int kv = lane >> 1, dh = lane & 1;
          tc::tma_load_3d(smem + kOffKV + st * 2 * kKVBytes + kv * kKVBytes + dh * (kKVBytes / 2),
                          kv ? &tm_v : &tm_k, &kv_full[st], dh * 64, it.g, row_base + kt * kT,
                          pol_kv);
        }
        if (++st == kStages) { st = 0; ph ^= 1; }
        if (j == 0) {
          if (kq > 0 && !tc::mbar_wait_warp(&q_free, (kq - 1) & 1, a.status)) { ok = false; break; }
          if (lane == 0) {
            tc::mbar_arrive_expect_tx(&q_full, it.nq * kQTileBytes);
            for (int t = 0; t < it.nq; ++t)
              for (int dh = 0; dh < 2; ++dh)
                tc::tma_load_3d(smem + kOffQ + t * kQTileBytes + dh * (kQTileBytes / 2), &tm_q,
                                &q_full, dh * 64, it.h0 + t, row_base + it.qt * kT,
                                tc::policy_evict_first());
          }
          __syncwarp();
        }
      }
      if (v.n > 0) ++kq;
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = tc::idesc_bf16_f32(128, kT);
      const uint32_t id_pv = tc::idesc_bf16_f32_bmn(128, kD);
      auto issue_qk = [&](int t, int st) {
        const uint32_t qaddr = sbase + kOffQ + t * kQTileBytes;
        const uint32_t kaddr = sbase + kOffKV + st * 2 * kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          tc::mma_bf16_ss(tmem + kColS + t * 128,
                          tc::sdesc_kmajor_sw128(qaddr + (kk >> 2) * (kQTileBytes / 2) + off),
                          tc::sdesc_kmajor_sw128(kaddr + (kk >> 2) * (kKVBytes / 2) + off), id_qk,
                          kk != 0);
        }
        tc::mma_commit(&s_full[t]);
      };
      int st = 0, kq = 0;
      uint32_t ph = 0;
      int steps[2] = {0, 0}, items_t[2] = {0, 0};  // per query tile: stages and items so far
      bool ok = true;
      for (int k = 0; k * n_ctas < a.n_items && ok; ++k) {
        const int i = item_index(k, cta, n_ctas, a.n_items);
        if (i < 0) continue;
        const Item it = item_of<kViews>(i, a);
        const VisRanges v = visible_ranges(it.qs, a);
        if (v.n == 0) continue;
        if (!tc::mbar_wait(&q_full, kq & 1, a.status) || !tc::mbar_wait(&kv_full[st], ph, a.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        for (int t = 0; t < it.nq; ++t) issue_qk(t, st);
        for (int j = 0; ok; ++j) {
          const bool more = j + 1 < v.n;
          // Q is read by no further product of this item once these are done
          if (!more && j == 0) tc::mma_commit(&q_free);
          const int st1 = st + 1 == kStages ? 0 : st + 1;
          const uint32_t ph1 = st + 1 == kStages ? ph ^ 1 : ph;
          const uint32_t vaddr = sbase + kOffKV + st * 2 * kKVBytes + kKVBytes;
          for (int t = 0; t < it.nq && ok; ++t) {
            if (!tc::mbar_wait(&p_full[t], (steps[t] + j) & 1, a.status)) { ok = false; break; }
            // the first product of an item overwrites O: the previous item's
            // O of this tile must have been read out
            if (j == 0 && items_t[t] > 0 && !tc::mbar_wait(&o_free[t], (items_t[t] - 1) & 1, a.status)) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kT / 16; ++kk)
              tc::mma_bf16_ts(tmem + kColO + t * 128, tmem + kColS + t * 128 + kk * 8,
                              tc::sdesc_mnmajor_sw128(vaddr + kk * 16 * 128, kKVBytes / 2), id_pv,
                              (j | kk) != 0);
            tc::mma_commit(&pv_done[t]);
            if (more) {
              if (t == 0 && !tc::mbar_wait(&kv_full[st1], ph1, a.status)) { ok = false; break; }
              tc::tc_fence_after();
              issue_qk(t, st1);
            }
          }
          if (!ok) break;
          // the products that read Q last have been issued: Q may be replaced once done
          if (j + 2 == v.n) tc::mma_commit(&q_free);
          tc::mma_commit(&kv_empty[st]);
          st = st1;
          ph = ph1;
          if (!more) {
            for (int t = 0; t < it.nq; ++t) {
              steps[t] += j + 1;
              ++items_t[t];
            }
            break;
          }
        }
        ++kq;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax / correction
    const int t = (warp - 4) / 4;
    const int q = warp & 3;
    const int r = 32 * q + lane;            // row within the query tile
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const float scale = kLog2e * rsqrtf(static_cast<float>(kD));
    const uint32_t sbuf = tmem + lane_off + kColS + t * 128;
    const uint32_t o_addr = tmem + lane_off + kColO + t * 128;
    uint8_t* stg = smem + kOffStg + (warp - 4) * 4096;  // this warp's 4 KB output box
    int steps = 0;        // stages of this query tile so far, over all items
    bool ok = true, stored = false;
    for (int k = 0; k * n_ctas < a.n_items && ok; ++k) {
      const int ii = item_index(k, cta, n_ctas, a.n_items);
      if (ii < 0) continue;
      const Item it = item_of<kViews>(ii, a);
      if (t >= it.nq) continue;
      const int i = it.qt * kT + r;         // absolute row in [0, 2L)
      float m = -INFINITY, l = 0.f;
      const VisRanges v = visible_ranges(it.qs, a);
      int j = 0;
      for (; j < v.n; ++j) {
        const int kt = vis_tile(v, j, a.n_qt / 2);
        const int kind = tile_visibility(it.qs, span_of(kt, a.L, a.D), a.D);
        if (!tc::mbar_wait_warp(&s_full[t], (steps + j) & 1, a.status)) { ok = false; break; }
        tc::tc_fence_after();
        uint32_t sr[128];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          tc::tmem_ld_32x32b_x32(sbuf + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
        tc::tmem_ld_wait();
        // Visible 32-key chunks of this key tile for this warp's rows (4 bits,
        // warp-uniform).  When D is a multiple of 32 a warp's 32 rows lie in
        // one block and so does each 32-key chunk, so a chunk is wholly
        // visible or wholly masked: masked chunks get no exponentials and P = 0.
        // Otherwise partly visible tiles are masked element by element.
        uint32_t cmask = 0xFu;
        if (kind != 2) {  // warp-uniform: partly visible key tile
          const int j0 = kt * kT;
          if (a.D % 32 == 0) {
            const int iw = it.qt * kT + 32 * q;  // the warp's first row
            cmask = 0u;
#pragma unroll
            for (int c = 0; c < 4; ++c) cmask |= pair_visible(iw, j0 + 32 * c, a.L, a.D) ? 1u << c : 0u;
          } else {
#pragma unroll
            for (int kk = 0; kk < 128; ++kk)
              if (!pair_visible(i, j0 + kk, a.L, a.D)) sr[kk] = __float_as_uint(-INFINITY);
          }
        }
        float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if ((cmask >> c) & 1u) {
#pragma unroll
            for (int kk = 32 * c; kk < 32 * c + 32; kk += 2)
              mk[(kk >> 1) & 3] = tc::fmax3(mk[(kk >> 1) & 3], __uint_as_float(sr[kk]), __uint_as_float(sr[kk + 1]));
          }
        const float mt = fmaxf(fmaxf(mk[0], mk[1]), fmaxf(mk[2], mk[3])) * scale;
        const float m_new = fmaxf(m, mt);
        // a row with no visible key in this tile keeps m = -inf until one shows up
        const bool rescale = (m == -INFINITY) || (m_new - m > kRescaleThreshold);
        float alpha = 1.f;
        if (rescale) {
          alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
          m = m_new;
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const float2 sc2 = make_float2(scale, scale), nm2 = make_float2(neg_m, neg_m);
        float2 rk[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if ((cmask >> c) & 1u) {
#pragma unroll
            for (int kk = 16 * c; kk < 16 * c + 16; ++kk) {  // packs in place: sr[kk] <- (p_2kk, p_2kk+1)
              // paired fp32 arithmetic; a quarter of the pairs' exponentials on
              // the FMA pipe, the rest on MUFU (which gives exact zeros for
              // masked, -inf, scores; poly_exp2x2 floors at 2^-126, so those
              // are zeroed)
              const float s0 = __uint_as_float(sr[2 * kk]), s1 = __uint_as_float(sr[2 * kk + 1]);
              const float2 x = ffma2(make_float2(s0, s1), sc2, nm2);
              float2 e;
              if ((kk & 3) == 3) {
                e = poly_exp2x2(x);
                e.x = s0 == -INFINITY ? 0.f : e.x;
                e.y = s1 == -INFINITY ? 0.f : e.y;
              } else {
                e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
              }
              rk[kk & 1] = fadd2(rk[kk & 1], e);
              sr[kk] = tc::pack_bf16x2(e.x, e.y);
            }
          } else {
#pragma unroll
            for (int kk = 16 * c; kk < 16 * c + 16; ++kk) sr[kk] = 0u;
          }
        }
        l = l * alpha + ((rk[0].x + rk[0].y) + (rk[1].x + rk[1].y));
        // S_t(j) complete also means tile t's earlier products (P V of stage
        // j - 1 included) have completed: none of tile t's MMAs is in flight.
        const bool need = rescale && j > 0;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? alpha : 1.f;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tc::tmem_ld_32x32b_x32(o_addr + cc * 32, ov);
            tc::tmem_ld_wait();
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) ov[kk] = __float_as_uint(__uint_as_float(ov[kk]) * f);
            tc::tmem_st_32x32b_x32(o_addr + cc * 32, ov);
          }
        }
        tc::tmem_st_32x32b_x32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tc::tmem_st_32x32b_x32(sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tc::tmem_st_wait();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      if (j == 0) continue;
      steps += j;
      // ------------------------------------------------------------ output
      // O / l (bf16) of the warp's 32 rows as two (64 d x 32 rows) boxes
      // through the warp's 4 KB box in shared memory (128-byte-swizzled
      // layout) and TMA tile stores.  Once the second half of O is in
      // registers the tile's O is released to the next item's products.
      if (!tc::mbar_wait_warp(&pv_done[t], (steps - 1) & 1, a.status)) { ok = false; break; }
      tc::tc_fence_after();
      const int h = it.h0 + t;
      const int row = it.n * 2 * a.L + it.qt * kT + 32 * q;
      // a clean tile's rows are the same in every view of its sample
      const int n_out = kViews && it.qt >= a.n_qt / 2 ? a.views : 1;
      const float inv = 1.f / l;
      auto stage_box = [&](const uint32_t (&ov)[64]) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 8 bf16 = one 16-byte chunk
          uint4 v;
          v.x = tc::pack_bf16x2(__uint_as_float(ov[8 * kk + 0]) * inv, __uint_as_float(ov[8 * kk + 1]) * inv);
          v.y = tc::pack_bf16x2(__uint_as_float(ov[8 * kk + 2]) * inv, __uint_as_float(ov[8 * kk + 3]) * inv);
          v.z = tc::pack_bf16x2(__uint_as_float(ov[8 * kk + 4]) * inv, __uint_as_float(ov[8 * kk + 5]) * inv);
          v.w = tc::pack_bf16x2(__uint_as_float(ov[8 * kk + 6]) * inv, __uint_as_float(ov[8 * kk + 7]) * inv);
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((kk ^ (lane & 7)) << 4)) = v;
        }
      };
      uint32_t ov[64];
      tc::tmem_ld_32x32b_x32(o_addr, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
      tc::tmem_ld_32x32b_x32(o_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
      tc::tmem_ld_wait();
      if (stored) {  // the previous item's last store has read the box
        if (lane == 0) tc::bulk_wait_read<0>();
        __syncwarp();
      }
      stage_box(ov);
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        for (int vw = 0; vw < n_out; ++vw) tc::tma_store_3d(&tm_out, stg, 0, h, row + vw * 2 * a.L);
        tc::bulk_commit();
      }
      tc::tmem_ld_32x32b_x32(o_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
      tc::tmem_ld_32x32b_x32(o_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
      tc::tmem_ld_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(&o_free[t]);
        tc::bulk_wait_read<0>();
      }
      __syncwarp();
      stage_box(ov);
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        for (int vw = 0; vw < n_out; ++vw) tc::tma_store_3d(&tm_out, stg, 64, h, row + vw * 2 * a.L);
        tc::bulk_commit();
      }
      stored = true;
    }
    if (stored && lane == 0) tc::bulk_wait_read<0>();
    __syncwarp();
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

// [rows][H][128] bf16 viewed as (d, head, row): box = box_rows rows of one
// head, 64 d elements wide, 128-byte swizzle (loads of 128-row tiles; tile
// stores of 32 output rows).
bool make_tmap_heads(CUtensorMap* m, const void* base, uint64_t rows, uint32_t heads,
                     uint32_t box_rows = kT) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), heads, rows};
  const cuuint64_t strides[2] = {kD * 2, static_cast<cuuint64_t>(heads) * kD * 2};
  const cuuint32_t box[3] = {64, 1, box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool mask_attn_tc_supported(const bd_attn_shape& sh, int L) {
  return sh.dtype == BD_BF16 && sh.head_dim == kD && L % kT == 0 && 2 * L / kT <= 62;
}

cudaError_t launch_mask_attn_tc(const bd_attn_shape& sh, const void* q, const void* k,
                                const void* v, void* out, int n_seqs, int L, int block,
                                int32_t* status, cudaStream_t st) {
  return launch_mask_attn_tc_views(sh, q, k, v, out, n_seqs, 1, L, block, status, st);
}

cudaError_t launch_mask_attn_tc_views(const bd_attn_shape& sh, const void* q, const void* k,
                                      const void* v, void* out, int n_seqs, int views, int L,
                                      int block, int32_t* status, cudaStream_t st) {
  if (views <= 0 || n_seqs % views != 0) return cudaErrorInvalidValue;
  const int Hq = sh.n_heads_q, Hkv = sh.n_heads_kv;
  const uint64_t rows = static_cast<uint64_t>(n_seqs) * 2 * L;
  CUtensorMap tm_q, tm_k, tm_v, tm_out;
  if (!make_tmap_heads(&tm_q, q, rows, Hq) || !make_tmap_heads(&tm_k, k, rows, Hkv) ||
      !make_tmap_heads(&tm_v, v, rows, Hkv) || !make_tmap_heads(&tm_out, out, rows, Hq, 32))
    return cudaErrorInvalidValue;
  MaskArgs a{};
  a.L = L;
  a.D = block;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.n_qt = 2 * L / kT;
  a.out = static_cast<bf16*>(out);
  a.status = status;
  // views == 1: the plain kernel, without the shared-view bookkeeping
  auto kern = views > 1 ? mask_attn_tc_kernel<true> : mask_attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  a.per_group = (a.G + 1) / 2;
  a.n_seqs = n_seqs;
  a.views = views;
  a.n_samples = n_seqs / views;
  const long long n_items =
      static_cast<long long>(a.n_qt / 2) * (n_seqs + a.n_samples) * a.per_group * Hkv;
  if (n_items <= 0 || n_items > (1LL << 30)) return cudaErrorInvalidValue;
  a.n_items = static_cast<int>(n_items);
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  // one persistent CTA per SM (one fits: 225 KB of shared memory, all of TMEM)
  const int grid = static_cast<int>(n_items < sms ? n_items : sms);
  kern<<<grid, kThreads, kSmemBytes, st>>>(tm_q, tm_k, tm_v, tm_out, a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd
