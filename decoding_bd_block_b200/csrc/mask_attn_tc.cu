// bd_block_mask_attn on the 5th-generation tensor cores (bf16, head_dim 128):
// attention of the training forward over [noisy x_t ; clean x_0] under the
// block-diffusion mixed mask ("Fast-dLLM v2: Efficient Block-Diffusion
// LLM", key design 2).  With blk(i) = (i mod L) / D a noisy query sees the
// noisy keys of its own block and the clean keys of earlier blocks; a clean
// query sees the clean keys of its own and earlier blocks.
//
// CTA = (128-row query tile, pair of query heads of one KV group, view).  The
// two heads are the kernel's two query tiles Q_0, Q_1 (TMA, shared memory);
// they read the same K/V.  Of the 2L/128 key tiles only those the mask leaves
// visible to the query tile are streamed (two 128-key K/V stages); a tile
// that is only partly visible is masked element by element in the softmax.
// Per key tile the MMA thread ping-pongs O_t += P_t V (TS MMA, P in TMEM) and
// S_t = Q_t K^T (SS MMA); one thread per query row runs the base-2 online
// softmax with lazy rescaling, as in attn_tc.cu.  Every key of a row is
// seen by one CTA, so O / l goes straight to the output.
#include "bd_common.cuh"
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
constexpr int kSmemBytes = kOffKV + kStages * 2 * kKVBytes + 1024;

struct MaskArgs {
  int L, D, Hq, Hkv, G;
  int n_qt;       // 2L / 128
  int per_group;  // query-head pairs per KV group: ceil(G / 2)
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

__global__ void __launch_bounds__(kThreads, 1)
    mask_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_out, MaskArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t q_full;
  __shared__ uint64_t kv_full[kStages], kv_empty[kStages];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ uint32_t tmem_slot;
  __shared__ uint8_t kv_list[64];   // visible key tiles of this query tile, in order
  __shared__ uint8_t kv_kind[64];   // 1: partial, 2: full

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Heaviest query tiles first over the whole grid (blockIdx.z, the
  // slowest-varying index, is the work rank): noisy query tile w and clean
  // query tile n_qt / 2 + w both see w + 1 key tiles, so the ranks take
  // them in pairs from the last w down.
  const int half = a.n_qt / 2, rank = blockIdx.z, wq = half - 1 - rank / 2;
  const int qt = (rank & 1) ? wq : half + wq;
  const int pr = blockIdx.x, n = blockIdx.y;
  const int g = pr / a.per_group;
  const int w = pr % a.per_group;
  const int h0 = g * a.G + 2 * w;                 // first head of the pair
  const int nq = (2 * w + 1 < a.G) ? 2 : 1;      // odd G: the last pair has one head
  const Span qs = span_of(qt, a.L, a.D);

  if (warp == 2) {
    // The key tiles visible to this query tile, in order: one lane per tile
    // (up to 63 tiles, two rounds), compacted with a ballot.
    int cnt = 0;
    for (int kt0 = 0; kt0 < a.n_qt; kt0 += 32) {
      const int kt = kt0 + lane;
      const int vis = kt < a.n_qt ? tile_visibility(qs, span_of(kt, a.L, a.D), a.D) : 0;
      const uint32_t any = __ballot_sync(0xffffffffu, vis != 0);
      if (vis) {
        const int at = cnt + __popc(any & ((1u << lane) - 1u));
        kv_list[at] = static_cast<uint8_t>(kt);
        kv_kind[at] = static_cast<uint8_t>(vis);
      }
      cnt += __popc(any);
    }
    if (lane == 0) kv_list[63] = static_cast<uint8_t>(cnt);
  }
  if (threadIdx.x == 0) {
    tc::mbar_init(&q_full, 1);
    for (int i = 0; i < kStages; ++i) {
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
    // The query tiles do not depend on anything else: their loads start
    // before the set-up barrier, overlapping the TMEM allocation.
    tc::prefetch_tmap(&tm_q);
    tc::mbar_arrive_expect_tx(&q_full, nq * kQTileBytes);
    for (int t = 0; t < nq; ++t)
      for (int dh = 0; dh < 2; ++dh)
        tc::tma_load_3d(smem + kOffQ + t * kQTileBytes + dh * (kQTileBytes / 2), &tm_q, &q_full,
                        dh * 64, h0 + t, n * 2 * a.L + qt * kT, tc::policy_evict_first());
  }
  if (warp == 1) tc::tmem_alloc(&tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t sbase = tc::smem_u32(smem);
  const int n_tiles = kv_list[63];
  const int row_base = n * 2 * a.L;  // first row of this view in the [N*2L] dimension

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
    }
    const uint64_t pol_kv = tc::policy_evict_last();  // K/V tiles are re-read by other CTAs
    int st = 0;
    uint32_t ph = 0;
    for (int j = 0; j < n_tiles; ++j) {
      if (!tc::mbar_wait_warp(&kv_empty[st], ph ^ 1, a.status)) break;
      if (lane == 0) tc::mbar_arrive_expect_tx(&kv_full[st], 2 * kKVBytes);
      __syncwarp();
      if (lane < 4) {  // lane = (K or V, d half)
        const int kv = lane >> 1, dh = lane & 1;
        tc::tma_load_3d(smem + kOffKV + st * 2 * kKVBytes + kv * kKVBytes + dh * (kKVBytes / 2),
                        kv ? &tm_v : &tm_k, &kv_full[st], dh * 64, g,
                        row_base + kv_list[j] * kT, pol_kv);
      }
      if (++st == kStages) { st = 0; ph ^= 1; }
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
      bool ok = n_tiles > 0 && tc::mbar_wait(&q_full, 0, a.status) &&
                tc::mbar_wait(&kv_full[0], 0, a.status);
      tc::tc_fence_after();
      for (int t = 0; t < nq && ok; ++t) issue_qk(t, 0);
      int st = 0;
      uint32_t ph = 0;
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int st1 = st + 1 == kStages ? 0 : st + 1;
        const uint32_t ph1 = st + 1 == kStages ? ph ^ 1 : ph;
        const bool more = j + 1 < n_tiles;
        const uint32_t vaddr = sbase + kOffKV + st * 2 * kKVBytes + kKVBytes;
        for (int t = 0; t < nq && ok; ++t) {
          if (!tc::mbar_wait(&p_full[t], j & 1, a.status)) { ok = false; break; }
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
        tc::mma_commit(&kv_empty[st]);
        st = st1;
        ph = ph1;
      }
    }
  } else if (warp >= 4 && (warp - 4) / 4 < nq) {
    // ------------------------------------------------ softmax / correction
    const int t = (warp - 4) / 4;
    const int q = warp & 3;
    const int r = 32 * q + lane;            // row within the query tile
    const int i = qt * kT + r;              // absolute row in [0, 2L)
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const float scale = kLog2e * rsqrtf(static_cast<float>(kD));
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    const uint32_t sbuf = tmem + lane_off + kColS + t * 128;
    for (int j = 0; j < n_tiles && ok; ++j) {
      if (!tc::mbar_wait_warp(&s_full[t], j & 1, a.status)) { ok = false; break; }
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
      if (kv_kind[j] != 2) {  // warp-uniform: partly visible key tile
        const int j0 = kv_list[j] * kT;
        if (a.D % 32 == 0) {
          const int iw = qt * kT + 32 * q;  // the warp's first row
          cmask = 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c) cmask |= pair_visible(iw, j0 + 32 * c, a.L, a.D) ? 1u << c : 0u;
        } else {
#pragma unroll
          for (int k = 0; k < 128; ++k)
            if (!pair_visible(i, j0 + k, a.L, a.D)) sr[k] = __float_as_uint(-INFINITY);
        }
      }
      float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if ((cmask >> c) & 1u) {
#pragma unroll
          for (int k = 32 * c; k < 32 * c + 32; k += 2)
            mk[(k >> 1) & 3] = tc::fmax3(mk[(k >> 1) & 3], __uint_as_float(sr[k]), __uint_as_float(sr[k + 1]));
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
          for (int k = 16 * c; k < 16 * c + 16; ++k) {  // packs in place: sr[k] <- (p_2k, p_2k+1)
            // paired fp32 arithmetic; a quarter of the pairs' exponentials on
            // the FMA pipe, the rest on MUFU (which gives exact zeros for
            // masked, -inf, scores; poly_exp2x2 floors at 2^-126, so those
            // are zeroed)
            const float s0 = __uint_as_float(sr[2 * k]), s1 = __uint_as_float(sr[2 * k + 1]);
            const float2 x = ffma2(make_float2(s0, s1), sc2, nm2);
            float2 e;
            if ((k & 3) == 3) {
              e = poly_exp2x2(x);
              e.x = s0 == -INFINITY ? 0.f : e.x;
              e.y = s1 == -INFINITY ? 0.f : e.y;
            } else {
              e = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            }
            rk[k & 1] = fadd2(rk[k & 1], e);
            sr[k] = tc::pack_bf16x2(e.x, e.y);
          }
        } else {
#pragma unroll
          for (int k = 16 * c; k < 16 * c + 16; ++k) sr[k] = 0u;
        }
      }
      l = l * alpha + ((rk[0].x + rk[0].y) + (rk[1].x + rk[1].y));
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
      tc::tmem_st_32x32b_x32(sbuf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tc::tmem_st_32x32b_x32(sbuf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[t]);
    }
    // ---------------------------------------------------------------- output
    if (ok && n_tiles > 0 && tc::mbar_wait_warp(&pv_done[t], (n_tiles - 1) & 1, a.status)) {
      // O / l (bf16) of the warp's 32 rows goes through its 8 KB slice of the
      // query tile's Q buffer (no MMA reads Q after the last P V), written in
      // the 128-byte-swizzled layout of two (64 d x 32 rows) boxes, and out by
      // TMA tile stores.
      tc::tc_fence_after();
      const int h = h0 + t;
      const uint32_t o_addr = tmem + lane_off + kColO + t * 128;
      const float inv = 1.f / l;
      uint8_t* stg = smem + kOffQ + t * kQTileBytes + q * 8192;
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
        const int row = row_base + qt * kT + 32 * q;
        tc::tma_store_3d(&tm_out, stg, 0, h, row);
        tc::tma_store_3d(&tm_out, stg + 4096, 64, h, row);
        tc::bulk_commit();
        tc::bulk_wait_read<0>();
      }
      __syncwarp();
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
  cudaFuncSetAttribute(mask_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kSmemBytes);
  a.per_group = (a.G + 1) / 2;
  mask_attn_tc_kernel<<<dim3(a.per_group * Hkv, n_seqs, a.n_qt), kThreads, kSmemBytes, st>>>(
      tm_q, tm_k, tm_v, tm_out, a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace bd
