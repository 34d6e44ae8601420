// bd_block_attn on CUDA cores (fp32 storage, and any shape the tensor-core
// path does not take).  Attention of the current 32-token block over
// [cached pages ; the block itself], bidirectional inside the block and over
// the whole prefix ("Fast-dLLM v2: Efficient Block-Diffusion LLM", overall
// framework and key design 3).
//
// Three launches:
//   1. attn_prep   rotate q and k of the block at positions P..P+31 and lay
//                  the block's K/V out as one extra page in the workspace;
//   2. attn_split  split-KV: CTA (chunk, q head, seq) streams its chunk of
//                  pages through shared memory and keeps an online softmax
//                  (max, sum, O) per query row, in base-2 exponent units;
//   3. attn_merge  combines the chunks' (m, l, O) per row.
#include "bd_common.cuh"
#include "mask_attn.cuh"

namespace bd {

// ------------------------------------------------------------- prep kernel
// 8 consecutive elements of a row, converted to fp32 (one 16-byte load for
// bf16, two for fp32; rows are 16-byte aligned).
struct Vec8 {
  float f[8];
};
__device__ __forceinline__ Vec8 load8(const bf16* p) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
  Vec8 r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    r.f[2 * i] = x.x;
    r.f[2 * i + 1] = x.y;
  }
  return r;
}
__device__ __forceinline__ Vec8 load8(const float* p) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  return Vec8{{a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w}};
}
__device__ __forceinline__ void store8(bf16* p, const Vec8& v) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v.f[2 * i], v.f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(float* p, const Vec8& v) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v.f[0], v.f[1], v.f[2], v.f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v.f[4], v.f[5], v.f[6], v.f[7]);
}

// grid (32, batch), 256 threads; one CTA per position t of sequence s.
// Rotated q -> ws_q [B][Hq][32][d]; rotated k_blk and v_blk -> ws_blk
// [B][2][Hkv][32][d] (a cache page of the current block).  Work items of 8
// elements: q and k items carry the 8 matching elements of both halves of
// the rotation pairs (j, j + d/2); v items are plain copies.  Each thread
// issues the loads of its first two items before the rotation table is
// built, so the item loads and the double-precision angles overlap.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_prep_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const int32_t* __restrict__ n_blocks, T* __restrict__ ws_q, T* __restrict__ ws_blk, int Hq,
    int Hkv, RopeFreq freq) {
  constexpr int C = D / 16;  // items per (head, row): 8-element groups of the first half
  __shared__ float cs[D / 2];
  __shared__ float sn[D / 2];
  griddep_wait();  // first kernel of the call: the caller's inputs are complete after this
  griddep_launch_dependents();
  const int t = blockIdx.x, s = blockIdx.y;
  const int n_q = Hq * C, n_k = Hkv * C, n_v = Hkv * 2 * C;
  const int total = n_q + n_k + n_v;
  const size_t row = static_cast<size_t>(s) * kBlock + t;
  // item -> (source, destination) of its (first) 8 elements
  auto src_of = [&](int it) -> const T* {
    if (it < n_q) return q + (row * Hq + it / C) * D + (it % C) * 8;
    it -= n_q;
    if (it < n_k) return k + (row * Hkv + it / C) * D + (it % C) * 8;
    it -= n_k;
    return v + (row * Hkv + it / (2 * C)) * D + (it % (2 * C)) * 8;
  };
  auto dst_of = [&](int it) -> T* {
    if (it < n_q) return ws_q + ((static_cast<size_t>(s) * Hq + it / C) * kBlock + t) * D + (it % C) * 8;
    it -= n_q;
    if (it < n_k)
      return ws_blk + ((static_cast<size_t>(s) * 2 + 0) * Hkv + it / C) * kBlock * D + t * D +
             (it % C) * 8;
    it -= n_k;
    return ws_blk + ((static_cast<size_t>(s) * 2 + 1) * Hkv + it / (2 * C)) * kBlock * D + t * D +
           (it % (2 * C)) * 8;
  };
  auto process = [&](int it, const Vec8& lo, const Vec8& hi) {
    T* dst = dst_of(it);
    if (it >= n_q + n_k) {
      store8(dst, lo);
      return;
    }
    const int j0 = (it % C) * 8;
    Vec8 a, b;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      a.f[e] = lo.f[e] * cs[j0 + e] - hi.f[e] * sn[j0 + e];
      b.f[e] = hi.f[e] * cs[j0 + e] + lo.f[e] * sn[j0 + e];
    }
    store8(dst, a);
    store8(dst + D / 2, b);
  };
  Vec8 lo[2], hi[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int it = threadIdx.x + u * blockDim.x;
    if (it < total) {
      const T* src = src_of(it);
      lo[u] = load8(src);
      if (it < n_q + n_k) hi[u] = load8(src + D / 2);
    }
  }
  const long long pos = static_cast<long long>(n_blocks[s]) * kBlock + t;
  for (int j = threadIdx.x; j < D / 2; j += blockDim.x) rope_cos_sin(pos, freq.inv[j], &cs[j], &sn[j]);
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int it = threadIdx.x + u * blockDim.x;
    if (it < total) process(it, lo[u], hi[u]);
  }
  for (int it = threadIdx.x + 2 * blockDim.x; it < total; it += blockDim.x) {
    const T* src = src_of(it);
    const Vec8 l = load8(src);
    process(it, l, it < n_q + n_k ? load8(src + D / 2) : l);
  }
}

// ----------------------------------------------------- split-KV CUDA-core
// One 32-key tile step of the online softmax for the 4 rows a warp owns.
// Qs: [32][D] pre-scaled by log2(e)/sqrt(D); Kt: [D][33] (transposed K);
// Vs: [32][D].  vis(r, lane) tells whether key `lane` is visible to row r.
template <int D, typename Vis>
__device__ __forceinline__ void simt_tile_step(const float* Qs, const float* Kt, const float* Vs,
                                               int warp, int lane, float (&m)[4], float (&l)[4],
                                               float (&o)[4][D / 32], Vis vis) {
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    float sc = 0.f;
#pragma unroll 16
    for (int c = 0; c < D; ++c) sc = fmaf(Qs[r * D + c], Kt[c * 33 + lane], sc);
    const bool ok = vis(r, lane);
    sc = ok ? sc : -INFINITY;
    const float mt = warp_max(sc);
    if (mt == -INFINITY) continue;  // warp-uniform: nothing visible in this tile
    const float mn = fmaxf(m[rr], mt);
    const float p = ok ? fast_exp2(sc - mn) : 0.f;
    const float alpha = (m[rr] == -INFINITY) ? 0.f : fast_exp2(m[rr] - mn);
    l[rr] = l[rr] * alpha + warp_sum(p);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o[rr][c] *= alpha;
#pragma unroll 8
    for (int j = 0; j < 32; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) o[rr][c] = fmaf(pj, Vs[j * D + lane + 32 * c], o[rr][c]);
    }
    m[rr] = mn;
  }
}

template <typename T, int D>
__device__ __forceinline__ void stage_kv(const T* kp, const T* vp, float* Kt, float* Vs) {
  for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) {
    const int j = i / D, c = i % D;
    Kt[c * 33 + j] = to_f32(kp[i]);
    Vs[i] = to_f32(vp[i]);
  }
}

// grid (max_chunks, Hq, batch), 256 threads (8 warps x 4 rows = 32 rows =
// the 32 positions of one query head).
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_split_simt_kernel(
    const T* __restrict__ pages, long long n_pages, const int32_t* __restrict__ page_table,
    int max_blocks, const int32_t* __restrict__ n_blocks, const T* __restrict__ ws_q,
    const T* __restrict__ ws_blk, float* __restrict__ part_o, float* __restrict__ part_ml,
    T* __restrict__ out, int Hq, int Hkv, int ppc, int max_chunks) {
  extern __shared__ float smem[];
  float* Qs = smem;             // [32][D]
  float* Kt = Qs + kBlock * D;  // [D][33]
  float* Vs = Kt + D * 33;      // [32][D]
  const int c = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int nb = min(max(n_blocks[s], 0), max_blocks);
  const int total = nb + 1;
  const int p0 = c * ppc;
  if (p0 >= total) return;
  const int p1 = min(total, p0 + ppc);
  const int g = h / (Hq / Hkv);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float qscale = kLog2e * rsqrtf(static_cast<float>(D));
  const T* qsrc = ws_q + (static_cast<size_t>(s) * Hq + h) * kBlock * D;
  for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) Qs[i] = to_f32(qsrc[i]) * qscale;

  float m[4], l[4], o[4][D / 32];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) o[rr][cc] = 0.f;
  }
  for (int p = p0; p < p1; ++p) {
    const T* kp;
    const T* vp;
    if (p < nb) {
      const int page = page_table[static_cast<size_t>(s) * max_blocks + p];
      if (threadIdx.x == 0) BD_CHECK(page >= 0 && page < n_pages, kCheckPageId, page);
      if (page < 0 || page >= n_pages) continue;  // CTA-uniform; host-validated
      kp = pages + ((static_cast<size_t>(page) * 2 + 0) * Hkv + g) * kBlock * D;
      vp = pages + ((static_cast<size_t>(page) * 2 + 1) * Hkv + g) * kBlock * D;
    } else {
      kp = ws_blk + ((static_cast<size_t>(s) * 2 + 0) * Hkv + g) * kBlock * D;
      vp = ws_blk + ((static_cast<size_t>(s) * 2 + 1) * Hkv + g) * kBlock * D;
    }
    __syncthreads();
    stage_kv<T, D>(kp, vp, Kt, Vs);
    __syncthreads();
    simt_tile_step<D>(Qs, Kt, Vs, warp, lane, m, l, o, [](int, int) { return true; });
  }

  const bool single = (total <= ppc) || (max_chunks == 1);
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    if (single) {
      const float inv = 1.f / l[rr];
      T* dst = out + ((static_cast<size_t>(s) * kBlock + r) * Hq + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) dst[lane + 32 * cc] = from_f32<T>(o[rr][cc] * inv);
    } else {
      const size_t row = ((static_cast<size_t>(s) * Hq + h) * max_chunks + c) * kBlock + r;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) part_o[row * D + lane + 32 * cc] = o[rr][cc];
      if (lane == 0) {
        part_ml[row * 2 + 0] = m[rr];
        part_ml[row * 2 + 1] = l[rr];
      }
    }
  }
}

// grid (kBlock / 8, Hq, batch), 256 threads: merge the chunks of 8 output
// rows of one query head, one warp per row.  Lane i holds the D / 32
// consecutive elements i * D / 32 ..: a warp reads a partial O row as one
// contiguous segment.  The chunks are taken eight at a time with all their
// loads in flight and folded into a running (max, sum, O) in base-2 exponent
// units, so a sequence of up to eight chunks costs one round trip to L2.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(const int32_t* __restrict__ n_blocks,
                                                         const float* __restrict__ part_o,
                                                         const float* __restrict__ part_ml,
                                                         T* __restrict__ out, int Hq, int ppc,
                                                         int max_chunks) {
  constexpr int E = D / 32;  // elements per lane
  static_assert(E == 2 || E == 4, "head_dim 64 or 128");
  constexpr int kGroup = 8;  // chunks in flight
  const int t = blockIdx.x * 8 + threadIdx.x / 32, h = blockIdx.y, s = blockIdx.z;
  const int d0 = (threadIdx.x % 32) * E;
  griddep_wait();  // the split kernel's partials
  griddep_launch_dependents();
  const int total = max(n_blocks[s], 0) + 1;
  if (total <= ppc) return;  // written directly by the split kernel
  const int nch = min((total + ppc - 1) / ppc, max_chunks);
  const size_t base = (static_cast<size_t>(s) * Hq + h) * max_chunks;
  const float2* ml = reinterpret_cast<const float2*>(part_ml);
  float M = -INFINITY, L = 0.f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int c0 = 0; c0 < nch; c0 += kGroup) {
    float2 v[kGroup];
    float o[kGroup][E];
#pragma unroll
    for (int u = 0; u < kGroup; ++u) {
      v[u] = make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int e = 0; e < E; ++e) o[u][e] = 0.f;
      if (c0 + u < nch) {
        const size_t r = (base + c0 + u) * kBlock + t;
        v[u] = ml[r];
        const float* src = part_o + r * D + d0;
        if constexpr (E == 4) {
          const float4 x = *reinterpret_cast<const float4*>(src);
          o[u][0] = x.x, o[u][1] = x.y, o[u][2] = x.z, o[u][3] = x.w;
        } else {
          const float2 x = *reinterpret_cast<const float2*>(src);
          o[u][0] = x.x, o[u][1] = x.y;
        }
      }
    }
    float Mn = M;
#pragma unroll
    for (int u = 0; u < kGroup; ++u) Mn = fmaxf(Mn, v[u].x);
    const float sc = M == -INFINITY ? 0.f : exp2f(M - Mn);
    L *= sc;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] *= sc;
#pragma unroll
    for (int u = 0; u < kGroup; ++u) {
      const float w = v[u].x == -INFINITY ? 0.f : exp2f(v[u].x - Mn);
      L = fmaf(v[u].y, w, L);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(o[u][e], w, acc[e]);
    }
    M = Mn;
  }
  const float inv = 1.f / L;
  T* dst = out + ((static_cast<size_t>(s) * kBlock + t) * Hq + h) * D + d0;
#pragma unroll
  for (int e = 0; e < E; ++e) dst[e] = from_f32<T>(acc[e] * inv);
}

// -------------------------------------------------------------- host side
// Tensor-core split: one CTA per SM at a time, so pick the chunk size (a
// multiple of 4 pages) that minimises waves x (pages per chunk + a fixed cost) over all (chunk, kv
// head, sequence) CTAs.  The fixed cost, worth ~8 pages of K/V traffic,
// stands for the CTA's query load (up to 64 KB), set-up and its fp32 partial
// (m, l, O) for the merge; at least 4 pages (two 64-key stages) per chunk.
static int plan_tc_chunk(const bd_attn_shape& sh, const bd_kv_cache& c, int max_pages) {
  int sms = 0, dev = 0;
  cudaGetDevice(&dev);
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  const int cap = attn_tc_max_chunk_pages();
  long long best_cost = -1;
  int best = cap;
  for (int ppc = 4; ppc <= cap; ppc += 4) {  // whole 128-key stages
    long long ctas = 0;
    for (int s = 0; s < c.batch; ++s) ctas += (c.n_blocks_host[s] + 1 + ppc - 1) / ppc;
    ctas *= sh.n_heads_kv;
    const long long cost = ((ctas + sms - 1) / sms) * static_cast<long long>(ppc + 8);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = ppc;
    }
    if (ppc >= max_pages) break;
  }
  return best;
}

AttnPlan plan_block_attn(const bd_attn_shape& sh, const bd_kv_cache& c) {
  AttnPlan p{};
  long long total_pages = 0;
  int max_pages = 1;
  for (int s = 0; s < c.batch; ++s) {
    total_pages += c.n_blocks_host[s] + 1;
    max_pages = max_pages > c.n_blocks_host[s] + 1 ? max_pages : c.n_blocks_host[s] + 1;
  }
  p.tc = attn_tc_supported(sh);
  long long ppc;
  if (p.tc) {
    ppc = plan_tc_chunk(sh, c, max_pages);
  } else {
    // About four CTAs per SM over all (chunk, q head, sequence) work items.
    const long long target = 4LL * 148;
    ppc = (total_pages * sh.n_heads_q + target - 1) / target;
    if (ppc < 1) ppc = 1;
    if (ppc > max_pages) ppc = max_pages;
  }
  p.pages_per_chunk = static_cast<int>(ppc);
  p.max_chunks = (max_pages + p.pages_per_chunk - 1) / p.pages_per_chunk;
  const size_t es = sh.dtype == BD_BF16 ? 2 : 4;
  const size_t d = sh.head_dim;
  size_t off = 0;
  p.off_q = off;
  off = align_up(off + static_cast<size_t>(c.batch) * sh.n_heads_q * kBlock * d * es, 256);
  p.off_blk = off;
  off = align_up(off + static_cast<size_t>(c.batch) * 2 * sh.n_heads_kv * kBlock * d * es, 256);
  const size_t rows = static_cast<size_t>(c.batch) * sh.n_heads_q * p.max_chunks * kBlock;
  p.off_o = off;
  off = align_up(off + (p.max_chunks > 1 ? rows * d * 4 : 0), 256);
  p.off_ml = off;
  off = align_up(off + (p.max_chunks > 1 ? rows * 2 * 4 : 0), 256);
  p.off_status = off;
  off = align_up(off + 4, 256);
  p.total = off;
  return p;
}

template <typename T, int D>
static cudaError_t launch_attn_t(const bd_attn_shape& sh, const bd_kv_cache& c, const AttnPlan& p,
                                 const void* q, const void* k, const void* v, void* out, void* ws,
                                 cudaStream_t st) {
  char* w = static_cast<char*>(ws);
  T* ws_q = reinterpret_cast<T*>(w + p.off_q);
  T* ws_blk = reinterpret_cast<T*>(w + p.off_blk);
  float* part_o = reinterpret_cast<float*>(w + p.off_o);
  float* part_ml = reinterpret_cast<float*>(w + p.off_ml);
  RopeFreq freq;
  rope_freq_table(D, sh.rope_theta, &freq);
  cudaError_t e = launch_pdl(attn_prep_kernel<T, D>, dim3(kBlock, c.batch), dim3(256), 0, st,
                             static_cast<const T*>(q), static_cast<const T*>(k),
                             static_cast<const T*>(v), c.n_blocks, ws_q, ws_blk, sh.n_heads_q,
                             sh.n_heads_kv, freq);
  if (e != cudaSuccess) return e;
  count_launches(1);
  if (p.tc) {
    e = launch_attn_tc(sh, c, p.pages_per_chunk, p.max_chunks, ws_q, ws_blk, part_o, part_ml, out,
                       reinterpret_cast<int32_t*>(w + p.off_status), st);
    if (e != cudaSuccess) return e;
    if (p.max_chunks > 1) {
      e = launch_pdl(attn_merge_kernel<T, D>, dim3(kBlock / 8, sh.n_heads_q, c.batch), dim3(256), 0, st,
                     c.n_blocks, part_o, part_ml, static_cast<T*>(out), sh.n_heads_q,
                     p.pages_per_chunk, p.max_chunks);
      if (e != cudaSuccess) return e;
      count_launches(1);
    }
    return cudaGetLastError();
  }
  const size_t smem = (kBlock * D + D * 33 + kBlock * D) * sizeof(float);
  auto kern = attn_split_simt_kernel<T, D>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  kern<<<dim3(p.max_chunks, sh.n_heads_q, c.batch), 256, smem, st>>>(
      static_cast<const T*>(c.pages), c.n_pages, c.page_table, c.max_blocks, c.n_blocks, ws_q,
      ws_blk, part_o, part_ml, static_cast<T*>(out), sh.n_heads_q, sh.n_heads_kv,
      p.pages_per_chunk, p.max_chunks);
  if (p.max_chunks > 1)
    attn_merge_kernel<T, D><<<dim3(kBlock / 8, sh.n_heads_q, c.batch), 256, 0, st>>>(
        c.n_blocks, part_o, part_ml, static_cast<T*>(out), sh.n_heads_q, p.pages_per_chunk,
        p.max_chunks);
  count_launches(p.max_chunks > 1 ? 2 : 1);
  return cudaGetLastError();
}

cudaError_t launch_block_attn(const bd_attn_shape& sh, const bd_kv_cache& c, const AttnPlan& p,
                              const void* q, const void* k, const void* v, void* out, void* ws,
                              cudaStream_t st) {
  const bool b = sh.dtype == BD_BF16;
  if (sh.head_dim == 64)
    return b ? launch_attn_t<bf16, 64>(sh, c, p, q, k, v, out, ws, st)
             : launch_attn_t<float, 64>(sh, c, p, q, k, v, out, ws, st);
  return b ? launch_attn_t<bf16, 128>(sh, c, p, q, k, v, out, ws, st)
           : launch_attn_t<float, 128>(sh, c, p, q, k, v, out, ws, st);
}

// ------------------------------------------------- 2L x 2L mask attention
// Visibility of key j to query i under the block-diffusion training mask
// ("Fast-dLLM v2", key design 2): rows/keys < L are the noisy stream x_t,
// the rest the clean stream x_0; blk(i) = (i mod L) / D.
__device__ __forceinline__ bool mixed_visible(int i, int j, int L, int D) {
  const bool qn = i < L, kn = j < L;
  const int bq = (qn ? i : i - L) / D, bk = (kn ? j : j - L) / D;
  if (qn) return kn ? (bk == bq) : (bk < bq);
  return kn ? false : (bk <= bq);
}

// grid (2L/32, Hq, n_seqs), 256 threads: 32 query rows of one head.
template <typename T, int D>
__global__ void __launch_bounds__(256) mask_attn_simt_kernel(const T* __restrict__ q,
                                                             const T* __restrict__ k,
                                                             const T* __restrict__ v,
                                                             T* __restrict__ out, int L, int blk,
                                                             int Hq, int Hkv) {
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Kt = Qs + kBlock * D;
  float* Vs = Kt + D * 33;
  const int qt = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int g = h / (Hq / Hkv);
  const int T2 = 2 * L;
  const int i0 = qt * kBlock;
  const bool qn = i0 < L;
  const int bq_lo = (qn ? i0 : i0 - L) / blk, bq_hi = (qn ? i0 + 31 : i0 + 31 - L) / blk;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float qscale = kLog2e * rsqrtf(static_cast<float>(D));
  for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) {
    const int r = i / D, c = i % D;
    Qs[i] = to_f32(q[((static_cast<size_t>(n) * T2 + i0 + r) * Hq + h) * D + c]) * qscale;
  }
  float m[4], l[4], o[4][D / 32];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) o[rr][cc] = 0.f;
  }
  for (int kt = 0; kt < T2 / kBlock; ++kt) {
    const int j0 = kt * kBlock;
    const bool kn = j0 < L;
    const int bk_lo = (kn ? j0 : j0 - L) / blk, bk_hi = (kn ? j0 + 31 : j0 + 31 - L) / blk;
    bool any;
    if (qn) any = kn ? (bk_hi >= bq_lo && bk_lo <= bq_hi) : (bk_lo < bq_hi);
    else any = kn ? false : (bk_lo <= bq_hi);
    if (!any) continue;
    __syncthreads();
    for (int i = threadIdx.x; i < kBlock * D; i += blockDim.x) {
      const int j = i / D, c = i % D;
      const size_t src = ((static_cast<size_t>(n) * T2 + j0 + j) * Hkv + g) * D + c;
      Kt[c * 33 + j] = to_f32(k[src]);
      Vs[i] = to_f32(v[src]);
    }
    __syncthreads();
    simt_tile_step<D>(Qs, Kt, Vs, warp, lane, m, l, o,
                      [&](int r, int ln) { return mixed_visible(i0 + r, j0 + ln, L, blk); });
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    const float inv = 1.f / l[rr];
    T* dst = out + ((static_cast<size_t>(n) * T2 + i0 + r) * Hq + h) * D;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) dst[lane + 32 * cc] = from_f32<T>(o[rr][cc] * inv);
  }
}

template <typename T, int D>
static cudaError_t launch_mask_t(const bd_attn_shape& sh, const void* q, const void* k,
                                 const void* v, void* out, int n_seqs, int L, int block,
                                 cudaStream_t st) {
  const size_t smem = (kBlock * D + D * 33 + kBlock * D) * sizeof(float);
  auto kern = mask_attn_simt_kernel<T, D>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  kern<<<dim3(2 * L / kBlock, sh.n_heads_q, n_seqs), 256, smem, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<T*>(out), L, block, sh.n_heads_q, sh.n_heads_kv);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_block_mask_attn(const bd_attn_shape& sh, const void* q, const void* k,
                                   const void* v, void* out, int n_seqs, int L, int block,
                                   cudaStream_t st) {
  return launch_block_mask_attn_views(sh, q, k, v, out, n_seqs, 1, L, block, st);
}

cudaError_t launch_block_mask_attn_views(const bd_attn_shape& sh, const void* q, const void* k,
                                         const void* v, void* out, int n_seqs, int views, int L,
                                         int block, cudaStream_t st) {
  if (mask_attn_tc_supported(sh, L))
    return launch_mask_attn_tc_views(sh, q, k, v, out, n_seqs, views, L, block, nullptr, st);
  const bool b = sh.dtype == BD_BF16;
  if (sh.head_dim == 64)
    return b ? launch_mask_t<bf16, 64>(sh, q, k, v, out, n_seqs, L, block, st)
             : launch_mask_t<float, 64>(sh, q, k, v, out, n_seqs, L, block, st);
  return b ? launch_mask_t<bf16, 128>(sh, q, k, v, out, n_seqs, L, block, st)
           : launch_mask_t<float, 128>(sh, q, k, v, out, n_seqs, L, block, st);
}

}  // namespace bd

#ifdef BD_DEVICE_CHECKS
namespace bd {
cudaError_t check_word_attn_simt(int* host2, bool reset) { return read_check_word(host2, reset); }
}  // namespace bd
#endif
