// fp_search.cu -- block mean pooling, pooled-score search with the max-based threshold, index
// emission, and the device-side index-list validator.
//
// FlashPrefill ("Instantaneous Pattern Discovery and Thresholding ..."), skill summary page:
//   "Stage 1: Block-Level Attention Approximation" -- block queries/keys are the means of the
//   tokens of each B-token block (partial last block: mean over the tokens it holds), block scores
//   are qbar . kbar / sqrt(d);
//   "Core Concept" item 3, "Dynamic Thresholding" -- one max reduction replaces sorting and
//   cumulative sums: block j of row i is kept iff p_ij >= tau * max_j p_ij with p the causal
//   softmax of the block scores; since p_ij / max_j p_ij = exp(s_ij - max_j s_ij) no sum is needed:
//   keep iff s_ij - m_i >= ln(tau). The sink block 0 and the diagonal block i are always kept;
//   "Physical Index Jumping" -- kept blocks become ascending index lists.
//
// Both kernels are bandwidth kernels: the pool kernel streams Q and K once from HBM with 16-byte
// loads (the dominant bytes); the search kernel reads the small pooled tensors (L2 resident),
// keeps the pooled scores in registers (never materialised), reduces the row max with warp
// shuffles and writes the lists with ballot/popc compaction.
#include <cuda_bf16.h>

#include "fp_internal.h"
#include "fp_seq.cuh"

namespace fp {

// ------------------------------------------------------------------------------------ pool ----
// Work item = (global block gb, 1024-element column chunk of the Q row or of the K row).
// 128 threads x 8 bf16 (one 16-byte load) per token; tokens unrolled by 8 for memory parallelism.
constexpr int kPoolThreads = 128;
constexpr int kPoolChunk = kPoolThreads * 8;

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += __uint_as_float(w[i] << 16);
    a[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 ld_stream_16(const uint16_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Sequence tables in dynamic shared memory, sized for the launch's sequence count (a few bytes for
// one sequence), so that the many small pool CTAs all stay resident.
__host__ __device__ inline size_t pool_smem_bytes(int num_seqs) { return (size_t)(4 * (num_seqs + 1) + 1) * 4; }

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const PoolParams p) {
  extern __shared__ int pool_tab[];
  const int S = p.seq.num_seqs, B = p.seq.block;
  int* s_cu = pool_tab;
  int* s_cb = s_cu + (S + 1);
  int* s_pb = s_cb + (S + 1);
  int* s_ckb = s_pb + (S + 1);
  int* s_ok = s_ckb + (S + 1);
  if (!build_seq_tables(p.seq, s_cu, s_cb, nullptr, nullptr, 0, 0, 0, s_ok, p.dev_status, s_pb, s_ckb)) return;
  // work items: (query block, Q column chunk) first, then (key block, K column chunk); the key
  // blocks of a sequence cover its cached prefix and its new tokens
  const long long q_items = (long long)p.seq.total_blocks * p.q_chunks;
  const long long items = q_items + (long long)p.seq.total_kv_blocks * p.k_chunks;
  for (long long w = blockIdx.x; w < items; w += gridDim.x) {
    const bool is_q = w < q_items;
    const long long wl = is_q ? w : w - q_items;
    const int chunks = is_q ? p.q_chunks : p.k_chunks;
    const int gb = (int)(wl / chunks);
    const int part = (int)(wl % chunks);
    long long r0;  // first source row of the block
    int n;         // tokens in the block
    if (is_q) {
      const int s = find_seq(s_cb, S, gb);
      const int t0 = s_cu[s] + (gb - s_cb[s]) * B;
      r0 = t0;
      n = min(B, s_cu[s + 1] - t0);
    } else {
      const int s = find_seq(s_ckb, S, gb);
      const int u0 = (gb - s_ckb[s]) * B;
      const int klen = s_pb[s] * B + (s_cu[s + 1] - s_cu[s]);
      n = min(B, klen - u0);
      r0 = kv_row(p.seq, s_cu, s, u0);  // the block's n rows are contiguous (pages hold whole blocks)
      if (r0 < 0) {
        if (threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
        continue;
      }
    }
    const int row = is_q ? p.q_row : p.k_row;
    const int col = part * kPoolChunk + threadIdx.x * 8;
    if (col >= row) continue;
    const uint16_t* src = (is_q ? p.q : p.k) + r0 * row + col;
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int t = 0;
    for (; t + 8 <= n; t += 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ld_stream_16(src + (long long)(t + u) * row);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc_bf16x8(a, v[u]);
    }
    for (; t < n; ++t) acc_bf16x8(a, ld_stream_16(src + (long long)t * row));
    const float inv_n = 1.0f / (float)n;
    float* dst = (is_q ? p.q_pool : p.k_pool) + (long long)gb * row + col;
    float4 o0 = make_float4(a[0] * inv_n, a[1] * inv_n, a[2] * inv_n, a[3] * inv_n);
    float4 o1 = make_float4(a[4] * inv_n, a[5] * inv_n, a[6] * inv_n, a[7] * inv_n);
    reinterpret_cast<float4*>(dst)[0] = o0;
    reinterpret_cast<float4*>(dst)[1] = o1;
  }
}

cudaError_t launch_pool(const PoolParams& p, int grid, cudaStream_t st) {
  pool_kernel<<<grid, kPoolThreads, pool_smem_bytes(p.seq.num_seqs), st>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------- search ----
// CTA tile = (sequence s, kv-head g, TI consecutive query blocks) -> 64 rows (q-head, block) that
// all share the pooled keys of kv-head g (GQA). Row r: head offset r % G, block offset r / G.
// Scores, row max / min, threshold and emission happen in this one kernel; the block-score matrix
// is never written to memory. Two CTAs fit on an SM.
// Pooled keys stream through shared memory in chunks of 64 blocks (cp.async, next chunk in flight).
// Warp w scores key blocks 8w..8w+7 of a chunk (broadcast shared reads) against rows 2l, 2l+1 of
// lane l (pooled queries transposed in shared memory).
// Pass 0 (tensor cores): approximate row max / min of the pooled scores with mma.sync bf16 on a
// two-term split of the fp32 operands (x = hi + lo; q.k ~ qh.kh + qh.kl + ql.kh) and a rigorous
// per-row error bound eps_i = 2^-14 * |q_i| * max_j |k_j| / sqrt(d) (the dropped terms and the
// fp32 accumulation are below 2^-15 * sum_d |q_d k_d| <= 2^-15 * |q| |k|). A row is certainly
// all-kept when (min - max) - 2 eps >= ln(tau); it is then written as 0..i.
// If any row of the tile is not certain, the tile takes the exact fp32 path:
// Pass 1: exact row max m_i and row min of s_ij over j <= i (scores stay in registers); if
// min - max >= ln(tau) every causal block passes (fp32 subtraction is monotonic, so this is the
// decision the per-block test would take) and the row is written as 0..i.
// Pass 2: recompute the exact scores, stage them in shared memory, and one warp per 8 rows emits
// the kept blocks in ascending order with ballot/popc compaction.
constexpr int kSearchThreads = 256;
constexpr int kSearchWarps = kSearchThreads / 32;
constexpr int kSearchRows = 64;
constexpr int kKChunk = 64;                  // key blocks per chunk (8 per warp)
constexpr int kQTStride = kSearchRows + 4;   // transposed pooled-query row stride (floats)
constexpr int kKStride = kHeadDim + 4;       // pooled-key row stride (floats), 16-byte aligned

// Shared memory: fixed part, then the sequence tables sized for this launch's sequence count.
// k[1] doubles as the pass-2 score tile (see the assert).
struct SearchSmem {
  float k[2][kKChunk][kKStride];             // pooled keys, natural layout, two buffers
  float qT[kHeadDim][kQTStride];             // pooled queries, [d][row]
  float red[2][kSearchWarps][kSearchRows];   // per-warp row max / min
  float qnorm[kSearchRows];                  // |q_row| (pass 0 error bound)
  int kmax_bits;                             // max |k_j| of the tile's keys, as float bits
  int ok;
  int need_pass2;
  int need_exact;
};
// Pass-0 operand views: split bf16 [hi/lo][row][kBfStride] in the qT region (queries) and in the
// key region (keys); the padded stride keeps the 32-bit fragment loads conflict free.
constexpr int kBfStride = kHeadDim + 8;
static_assert(2 * kSearchRows * kBfStride * 2 <= (int)sizeof(float) * kHeadDim * kQTStride, "query split view");
static_assert(2 * kKChunk * kBfStride * 2 <= (int)sizeof(float) * 2 * kKChunk * kKStride, "key split view");
static_assert(kSearchRows * (kKChunk + 1) <= kKChunk * kKStride, "score tile must fit in one key buffer");

__host__ __device__ inline size_t search_smem_bytes(int num_seqs) {
  return sizeof(SearchSmem) + (size_t)(num_seqs + 1) * (5 * sizeof(int)) + 8 + (size_t)(num_seqs + 1) * 8;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_u32(dst);
  const int n = valid ? 16 : 0;  // 0 source bytes -> 16 zero bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all_but_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Issue the copies of chunk [j0, j0+64) of kv-head g's pooled keys into buffer `buf` (zero past jmax).
__device__ __forceinline__ void issue_k_chunk(SearchSmem& sm, int buf, const float* kp, int gb0, int g, int hkv,
                                              int j0, int jmax) {
  for (int e = threadIdx.x; e < kKChunk * (kHeadDim / 4); e += kSearchThreads) {
    const int jr = e / (kHeadDim / 4), c4 = e % (kHeadDim / 4);
    const int j = min(j0 + jr, jmax);
    cp_async16(&sm.k[buf][jr][4 * c4], kp + ((long long)(gb0 + j) * hkv + g) * kHeadDim + 4 * c4, j0 + jr <= jmax);
  }
  cp_async_commit();
}

// acc[e][b] = q_row(2*lane+e) . k_block(8*warp+b) over the full head dim.
__device__ __forceinline__ void chunk_scores(const SearchSmem& sm, int buf, int warp, int lane, float (&acc)[2][8]) {
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[e][b] = 0.f;
#pragma unroll 2
  for (int d = 0; d < kHeadDim; d += 4) {
    float4 kv[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) kv[b] = *reinterpret_cast<const float4*>(&sm.k[buf][8 * warp + b][d]);
#pragma unroll
    for (int dd = 0; dd < 4; ++dd) {
      const float2 q2 = *reinterpret_cast<const float2*>(&sm.qT[d + dd][2 * lane]);
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const float kk = dd == 0 ? kv[b].x : dd == 1 ? kv[b].y : dd == 2 ? kv[b].z : kv[b].w;
        acc[0][b] = fmaf(q2.x, kk, acc[0][b]);
        acc[1][b] = fmaf(q2.y, kk, acc[1][b]);
      }
    }
  }
}

__device__ __forceinline__ uint32_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// Split 4 fp32 values into bf16 hi and lo (x - hi) and store them at hi_dst / lo_dst (8 bytes each).
__device__ __forceinline__ void split_store4(uint16_t* hi_dst, uint16_t* lo_dst, float4 v) {
  const float x[4] = {v.x, v.y, v.z, v.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    h[e] = bf16_bits(x[e]);
    l[e] = bf16_bits(x[e] - __uint_as_float(h[e] << 16));
  }
  *reinterpret_cast<uint2*>(hi_dst) = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
  *reinterpret_cast<uint2*>(lo_dst) = make_uint2(l[0] | (l[1] << 16), l[2] | (l[3] << 16));
}

// 64 rows x 128 fp32 (rows via row_ptr) -> split bf16 view; optional per-row norms.
// Warp w handles rows w, w + 8, ...; lane l the 4 columns 4l..4l+3.
template <typename RowPtr>
__device__ __forceinline__ void load_split_rows(uint16_t* view, RowPtr row_ptr, float* norms, int* max_bits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kPer = kSearchRows / kSearchWarps;
  float4 vv[kPer];  // all loads in flight before any use (L2 latency paid once)
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const float* src = row_ptr(warp + q * kSearchWarps);
    vv[q] = src ? reinterpret_cast<const float4*>(src)[lane] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int r = warp + q * kSearchWarps;
    const float4 v = vv[q];
    split_store4(view + r * kBfStride + 4 * lane, view + (kSearchRows + r) * kBfStride + 4 * lane, v);
    float ss = v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      const float nrm = sqrtf(ss);
      if (norms) norms[r] = nrm;
      if (max_bits) atomicMax(max_bits, __float_as_int(nrm));
    }
  }
}

// Pass-0 key staging: fp32 chunk [64 rows][128] (unpadded) in the upper half of the key region, filled
// by cp.async while the previous chunk's MMAs run.
constexpr int kStageOffBytes = 2 * kKChunk * kBfStride * 2;
static_assert(kStageOffBytes + kKChunk * kHeadDim * 4 <= (int)sizeof(float) * 2 * kKChunk * kKStride, "staging");

__device__ __forceinline__ void issue_stage_chunk(float* stage, const float* kp, int gb0, int g, int hkv, int j0,
                                                  int jmax) {
  for (int e = threadIdx.x; e < kKChunk * (kHeadDim / 4); e += kSearchThreads) {
    const int jr = e / (kHeadDim / 4), c4 = e % (kHeadDim / 4);
    const int j = min(j0 + jr, jmax);
    cp_async16(stage + jr * kHeadDim + 4 * c4, kp + ((long long)(gb0 + j) * hkv + g) * kHeadDim + 4 * c4,
               j0 + jr <= jmax);
  }
  cp_async_commit();
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Pass-0 scores of one 64-block chunk: warp w covers rows 16(w%4).. and key blocks 32(w/4)..;
// acc[nt][e]: rows r0+g (e = 0,1) and r0+g+8 (e = 2,3), key blocks n0+8nt+2t+(e&1).
__device__ __forceinline__ void chunk_scores_tc(const uint16_t* qv, const uint16_t* kv, int warp, int lane,
                                                float (&acc)[4][4]) {
  const int g = lane >> 2, t = lane & 3;
  const int r0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  auto w32 = [](const uint16_t* base, int row, int col) {
    return *reinterpret_cast<const uint32_t*>(base + row * kBfStride + col);
  };
  const uint16_t* qh = qv;
  const uint16_t* ql = qv + kSearchRows * kBfStride;
  const uint16_t* kh = kv;
  const uint16_t* kl = kv + kKChunk * kBfStride;
#pragma unroll 2
  for (int kk = 0; kk < kHeadDim; kk += 16) {
    const int c0 = kk + 2 * t;
    const uint32_t ah[4] = {w32(qh, r0 + g, c0), w32(qh, r0 + g + 8, c0), w32(qh, r0 + g, c0 + 8), w32(qh, r0 + g + 8, c0 + 8)};
    const uint32_t al[4] = {w32(ql, r0 + g, c0), w32(ql, r0 + g + 8, c0), w32(ql, r0 + g, c0 + 8), w32(ql, r0 + g + 8, c0 + 8)};
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int n = n0 + 8 * nt + g;
      const uint32_t bh0 = w32(kh, n, c0), bh1 = w32(kh, n, c0 + 8);
      const uint32_t bl0 = w32(kl, n, c0), bl1 = w32(kl, n, c0 + 8);
      mma_bf16_16816(acc[nt], ah, bh0, bh1);
      mma_bf16_16816(acc[nt], ah, bl0, bl1);
      mma_bf16_16816(acc[nt], al, bh0, bh1);
    }
  }
}

__global__ void __launch_bounds__(kSearchThreads, 2) search_kernel(const SearchParams p) {
  extern __shared__ __align__(16) unsigned char search_smem_raw[];
  SearchSmem& sm = *reinterpret_cast<SearchSmem*>(search_smem_raw);
  const int S = p.seq.num_seqs;
  int* t_cu = reinterpret_cast<int*>(search_smem_raw + sizeof(SearchSmem));
  int* t_cb = t_cu + (S + 1);
  int* t_ct = t_cb + (S + 1);
  int* t_pb = t_ct + (S + 1);
  int* t_ckb = t_pb + (S + 1);
  long long* t_ib = reinterpret_cast<long long*>(((uintptr_t)(t_ckb + (S + 1)) + 7) & ~(uintptr_t)7);
  if (!build_seq_tables(p.seq, t_cu, t_cb, t_ct, t_ib, p.hq, p.rows_blocks * p.seq.block, p.hkv, &sm.ok,
                        p.dev_status, t_pb, t_ckb))
    return;
  if (t_ib[S] != p.index_elems) {
    if (blockIdx.x == 0 && threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
    return;
  }
  const int G = p.group, TI = p.rows_blocks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NB = p.seq.total_blocks;
  const unsigned lt_mask = (1u << lane) - 1u;

  const int num_tiles = t_ct[S];
  // boustrophedon over the grid: tiles are heaviest first, so alternating direction per round
  // balances the per-CTA work without a work queue
  for (int kr = 0;; ++kr) {
    const int tile = kr * gridDim.x + ((kr & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
    if (tile >= num_tiles) break;
    const int s = find_seq(t_ct, S, tile);
    const int local = tile - t_ct[s];
    const int nb = t_cb[s + 1] - t_cb[s];
    const int ntiles = (nb + TI - 1) / TI;
    const int it = ntiles - 1 - local / p.hkv;  // heavy (late) query blocks first
    const int g = local % p.hkv;
    const int i0 = it * TI;
    const int i_last = min(i0 + TI, nb) - 1;
    const int gb0 = t_cb[s];   // global query block of local block 0 (pooled queries, counts)
    const int pb = t_pb[s];    // cached prefix blocks: query block i is key block pb + i
    const int kb0 = t_ckb[s];  // global key block of the sequence's key block 0 (pooled keys)
    const int jmax = pb + i_last;  // last key block any row of the tile attends
    const int nchunks = jmax / kKChunk + 1;

    __syncthreads();  // previous tile done with shared memory
    const float* q_src = p.q_pool;  // pooled queries of the tile (global, L2 resident)
    auto q_row = [&](int r) -> const float* {
      const int i = i0 + r / G;
      return (r < TI * G && i <= i_last) ? q_src + ((long long)(gb0 + i) * p.hq + g * G + r % G) * kHeadDim : nullptr;
    };
    if (threadIdx.x == 0) {
      sm.need_pass2 = 0;
      sm.need_exact = 0;
      sm.kmax_bits = 0;
    }

    // emission rows: warp w emits rows 8w..8w+7; row_i is the local query block, row_j the last
    // key block of the row (its diagonal, pb + i), -1 for padding rows
    int row_i[8], row_j[8], row_h[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int rr = warp * 8 + r;
      row_i[r] = (rr < TI * G && i0 + rr / G <= i_last) ? i0 + rr / G : -1;
      row_j[r] = row_i[r] >= 0 ? pb + row_i[r] : -1;
      row_h[r] = g * G + rr % G;
    }
    bool all_keep[8];
    float rmx[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) { all_keep[r] = true; rmx[r] = 0.f; }

    if (!p.keep_all) {
      // ---- pass 0: approximate max / min on tensor cores, with a rigorous error bound
      uint16_t* qv = reinterpret_cast<uint16_t*>(&sm.qT[0][0]);
      uint16_t* kvw = reinterpret_cast<uint16_t*>(&sm.k[0][0][0]);
      __syncthreads();
      load_split_rows(qv, q_row, sm.qnorm, nullptr);
      const int g4 = lane >> 2, t4 = lane & 3;
      const int r0 = 16 * (warp & 3), n0 = 32 * (warp >> 2);
      int ri[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int r = r0 + g4 + 8 * h2;
        ri[h2] = (r < TI * G && i0 + r / G <= i_last) ? pb + i0 + r / G : -1;
      }
      float am[2] = {-INFINITY, -INFINITY}, an[2] = {INFINITY, INFINITY};
      float* stage = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(kvw) + kStageOffBytes);
      issue_stage_chunk(stage, p.k_pool, kb0, g, p.hkv, 0, jmax);
      for (int j0 = 0; j0 <= jmax; j0 += kKChunk) {
        cp_async_wait_all();
        __syncthreads();  // staged chunk visible; previous chunk's MMAs done with the split view
        load_split_rows(kvw, [&](int jr) -> const float* { return stage + jr * kHeadDim; }, nullptr,
                        &sm.kmax_bits);
        __syncthreads();  // split view ready; staging free
        if (j0 + kKChunk <= jmax) issue_stage_chunk(stage, p.k_pool, kb0, g, p.hkv, j0 + kKChunk, jmax);
        float acc[4][4];
        chunk_scores_tc(qv, kvw, warp, lane, acc);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = j0 + n0 + 8 * nt + 2 * t4 + (e & 1);
            const int h2 = e >> 1;
            if (j <= ri[h2]) {
              const float sc = acc[nt][e] * p.inv_sqrt_d;
              am[h2] = fmaxf(am[h2], sc);
              an[h2] = fminf(an[h2], sc);
            }
          }
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
          am[h2] = fmaxf(am[h2], __shfl_xor_sync(0xffffffffu, am[h2], o));
          an[h2] = fminf(an[h2], __shfl_xor_sync(0xffffffffu, an[h2], o));
        }
        if (t4 == 0) {
          sm.red[0][warp >> 2][r0 + g4 + 8 * h2] = am[h2];
          sm.red[1][warp >> 2][r0 + g4 + 8 * h2] = an[h2];
        }
      }
      __syncthreads();
      const float kmax = __int_as_float(sm.kmax_bits);
      bool uncertain = false;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int rr = warp * 8 + r;
        const float a = fmaxf(sm.red[0][0][rr], sm.red[0][1][rr]);
        const float b = fminf(sm.red[1][0][rr], sm.red[1][1][rr]);
        const float eps = 6.103515625e-05f * sm.qnorm[rr] * kmax * p.inv_sqrt_d;  // 2^-14 |q| max|k| / sqrt(d)
        if (row_i[r] >= 0 && !((b - a) - 2.f * eps >= p.log_tau)) uncertain = true;
      }
      if (uncertain && lane == 0) atomicOr(&sm.need_exact, 1);
      __syncthreads();

      if (sm.need_exact) {
        // ---- exact fp32 path for this tile
        for (int e = threadIdx.x; e < kSearchRows * (kHeadDim / 4); e += kSearchThreads) {
          const int r = e % kSearchRows, d4 = e / kSearchRows;
          const float* src = q_row(r);
          const float4 v = src ? reinterpret_cast<const float4*>(src)[d4] : make_float4(0.f, 0.f, 0.f, 0.f);
          sm.qT[4 * d4 + 0][r] = v.x;
          sm.qT[4 * d4 + 1][r] = v.y;
          sm.qT[4 * d4 + 2][r] = v.z;
          sm.qT[4 * d4 + 3][r] = v.w;
        }
        issue_k_chunk(sm, 0, p.k_pool, kb0, g, p.hkv, 0, jmax);
        // scoring rows of this lane (li: the row's last key block)
        int li[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = 2 * lane + e;
          li[e] = (r < TI * G && i0 + r / G <= i_last) ? pb + i0 + r / G : -1;
        }
        float mx[2] = {-INFINITY, -INFINITY}, mn[2] = {INFINITY, INFINITY};
        // ---- pass 1: exact row max / min of the pooled scores
        for (int c = 0; c < nchunks; ++c) {
          const int j0 = c * kKChunk;
          if (c + 1 < nchunks) {
            __syncthreads();  // buffer (c+1)&1 no longer read
            issue_k_chunk(sm, (c + 1) & 1, p.k_pool, kb0, g, p.hkv, j0 + kKChunk, jmax);
            cp_async_wait_all_but_one();
          } else {
            cp_async_wait_all();
          }
          __syncthreads();
          float acc[2][8];
          chunk_scores(sm, c & 1, warp, lane, acc);
#pragma unroll
          for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int b = 0; b < 8; ++b) {
              if (j0 + 8 * warp + b <= li[e]) {
                const float sc = acc[e][b] * p.inv_sqrt_d;
                mx[e] = fmaxf(mx[e], sc);
                mn[e] = fminf(mn[e], sc);
              }
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          sm.red[0][warp][2 * lane + e] = mx[e];
          sm.red[1][warp][2 * lane + e] = mn[e];
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int rr = warp * 8 + r;
          float a = -INFINITY, b = INFINITY;
#pragma unroll
          for (int w = 0; w < kSearchWarps; ++w) {
            a = fmaxf(a, sm.red[0][w][rr]);
            b = fminf(b, sm.red[1][w][rr]);
          }
          rmx[r] = a;
          all_keep[r] = (b - a >= p.log_tau);
        }
      }
    }
    bool warp_needs = false;
#pragma unroll
    for (int r = 0; r < 8; ++r)
      if (row_i[r] >= 0 && !all_keep[r]) warp_needs = true;
    const int warp_jmax = max(max(max(row_j[0], row_j[1]), max(row_j[2], row_j[3])),
                              max(max(row_j[4], row_j[5]), max(row_j[6], row_j[7])));
    if (warp_needs && lane == 0) atomicOr(&sm.need_pass2, 1);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (row_i[r] < 0 || !all_keep[r]) continue;
      const int i = row_i[r], jl = row_j[r];
      int32_t* dst = p.indices + list_row(t_cb, t_ib, t_pb, s, row_h[r], i);
      for (int j = lane; j <= jl; j += 32) dst[j] = j;
      if (lane == 0) p.counts[(long long)row_h[r] * NB + gb0 + i] = jl + 1;
    }
    __syncthreads();
    if (!sm.need_pass2) continue;

    // ---- pass 2: recompute the scores and emit kept blocks in ascending order
    float(*sc)[kKChunk + 1] = reinterpret_cast<float(*)[kKChunk + 1]>(&sm.k[1][0][0]);
    int cnt[8];
    int64_t base[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      cnt[r] = 0;
      base[r] = (row_i[r] >= 0) ? list_row(t_cb, t_ib, t_pb, s, row_h[r], row_i[r]) : 0;
    }
    for (int c = 0; c < nchunks; ++c) {
      const int j0 = c * kKChunk;
      __syncthreads();
      issue_k_chunk(sm, 0, p.k_pool, kb0, g, p.hkv, j0, jmax);
      cp_async_wait_all();
      __syncthreads();
      float acc[2][8];
      chunk_scores(sm, 0, warp, lane, acc);
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int b = 0; b < 8; ++b) sc[2 * lane + e][8 * warp + b] = acc[e][b] * p.inv_sqrt_d;
      __syncthreads();
      if (!warp_needs || j0 > warp_jmax) continue;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (row_i[r] < 0 || all_keep[r] || j0 > row_j[r]) continue;
#pragma unroll
        for (int h2 = 0; h2 < kKChunk; h2 += 32) {
          const int j = j0 + h2 + lane;
          const float v = sc[warp * 8 + r][h2 + lane];
          const bool keep = j <= row_j[r] && (j == 0 || j == row_j[r] || v - rmx[r] >= p.log_tau);
          const unsigned bal = __ballot_sync(0xffffffffu, keep);
          if (keep) p.indices[base[r] + cnt[r] + __popc(bal & lt_mask)] = j;
          cnt[r] += __popc(bal);
        }
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (row_i[r] >= 0 && !all_keep[r]) p.counts[(long long)row_h[r] * NB + gb0 + row_i[r]] = cnt[r];
    }
  }
}

cudaError_t launch_search(const SearchParams& p, cudaStream_t st) {
  static bool attr_done = false;
  const int smem = (int)search_smem_bytes(p.seq.num_seqs);
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(search_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)search_smem_bytes(kMaxSeqs));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cap = 2 * sms;
  const int grid = p.num_tiles < cap ? p.num_tiles : cap;
  if (grid <= 0) return cudaSuccess;
  search_kernel<<<grid, kSearchThreads, smem, st>>>(p);
  return cudaGetLastError();
}

// --------------------------------------------------------------------- top-p (comparison) ----
// The cumulative-probability selector the max-based threshold replaces (FlashPrefill skill summary
// page, "The Problem": Top-k / Top-p need score computation, sorting and cumulative sums;
// FlexPrefill abstract, "Cumulative-Attention Based Index Selection"). Built to measure its cost
// on the same pooled tensors: row (h, i) keeps block j iff the probability mass of the blocks that
// are strictly more probable than j is below gamma (ties at the cut kept together), plus the sink
// and the diagonal. It needs every score of a row before any decision, so it runs in two launches:
// 1. topp_score_kernel writes the exact fp32 pooled scores into a scratch buffer laid out like the
//    index lists (the score matrix the threshold search never materialises);
// 2. topp_select_kernel, one warp per row: the row max, e_j = exp(s_j - max) and Z = sum e_j; then
//    the cut x* = the smallest float x with F(x) = sum_{e_l > x} e_l < gamma * Z, found by
//    bisection on the float bits (F is non-increasing, 0 <= e <= 1); block j is kept iff e_j >= x*
//    (equivalently F(e_j) < gamma * Z); ascending emission with ballot/popc.
__global__ void __launch_bounds__(kSearchThreads, 2) topp_score_kernel(const SearchParams p, float* scores) {
  extern __shared__ __align__(16) unsigned char search_smem_raw[];
  SearchSmem& sm = *reinterpret_cast<SearchSmem*>(search_smem_raw);
  const int S = p.seq.num_seqs;
  int* t_cu = reinterpret_cast<int*>(search_smem_raw + sizeof(SearchSmem));
  int* t_cb = t_cu + (S + 1);
  int* t_ct = t_cb + (S + 1);
  int* t_pb = t_ct + (S + 1);
  int* t_ckb = t_pb + (S + 1);
  long long* t_ib = reinterpret_cast<long long*>(((uintptr_t)(t_ckb + (S + 1)) + 7) & ~(uintptr_t)7);
  if (!build_seq_tables(p.seq, t_cu, t_cb, t_ct, t_ib, p.hq, p.rows_blocks * p.seq.block, p.hkv, &sm.ok,
                        p.dev_status, t_pb, t_ckb))
    return;
  if (t_ib[S] != p.index_elems) {
    if (blockIdx.x == 0 && threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
    return;
  }
  const int G = p.group, TI = p.rows_blocks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = t_ct[S];
  for (int kr = 0;; ++kr) {
    const int tile = kr * gridDim.x + ((kr & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
    if (tile >= num_tiles) break;
    const int s = find_seq(t_ct, S, tile);
    const int local = tile - t_ct[s];
    const int nb = t_cb[s + 1] - t_cb[s];
    const int ntiles = (nb + TI - 1) / TI;
    const int it = ntiles - 1 - local / p.hkv;
    const int g = local % p.hkv;
    const int i0 = it * TI;
    const int i_last = min(i0 + TI, nb) - 1;
    const int gb0 = t_cb[s], pb = t_pb[s], kb0 = t_ckb[s];
    const int jmax = pb + i_last;
    const int nchunks = jmax / kKChunk + 1;
    __syncthreads();  // previous tile done with shared memory
    for (int e = threadIdx.x; e < kSearchRows * (kHeadDim / 4); e += kSearchThreads) {
      const int r = e % kSearchRows, d4 = e / kSearchRows;
      const int i = i0 + r / G;
      const bool ok = r < TI * G && i <= i_last;
      const float4 v = ok ? reinterpret_cast<const float4*>(
                                p.q_pool + ((long long)(gb0 + i) * p.hq + g * G + r % G) * kHeadDim)[d4]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      sm.qT[4 * d4 + 0][r] = v.x;
      sm.qT[4 * d4 + 1][r] = v.y;
      sm.qT[4 * d4 + 2][r] = v.z;
      sm.qT[4 * d4 + 3][r] = v.w;
    }
    // this lane's rows 2*lane + e: list start and last key block (-1: padding row)
    int64_t rbase[2];
    int rj[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 2 * lane + e;
      const int i = i0 + r / G;
      const bool ok = r < TI * G && i <= i_last;
      rj[e] = ok ? pb + i : -1;
      rbase[e] = ok ? list_row(t_cb, t_ib, t_pb, s, g * G + r % G, i) : 0;
    }
    issue_k_chunk(sm, 0, p.k_pool, kb0, g, p.hkv, 0, jmax);
    for (int c = 0; c < nchunks; ++c) {
      const int j0 = c * kKChunk;
      if (c + 1 < nchunks) {
        __syncthreads();  // buffer (c+1)&1 no longer read
        issue_k_chunk(sm, (c + 1) & 1, p.k_pool, kb0, g, p.hkv, j0 + kKChunk, jmax);
        cp_async_wait_all_but_one();
      } else {
        cp_async_wait_all();
      }
      __syncthreads();
      float acc[2][8];
      chunk_scores(sm, c & 1, warp, lane, acc);
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const int j = j0 + 8 * warp + b;
          if (j <= rj[e]) scores[rbase[e] + j] = acc[e][b] * p.inv_sqrt_d;
        }
    }
  }
}

struct ToppParams {
  SeqInfo seq;
  int32_t hq;
  float gamma;
  const float* scores;   // row (s, h, i) at the index-list row start, pb + i + 1 entries
  int32_t* counts;       // [Hq, NB]
  int32_t* indices;
  int64_t index_elems;
  int32_t* dev_status;
};

constexpr int kToppPer = 32;  // scores per lane held in registers (rows of up to 1024 blocks)

// F(x) = sum of e_l > x over the row (warp-wide), e in registers or re-read from the scratch
__device__ __forceinline__ float topp_mass_above(const float (&e)[kToppPer], bool in_regs, const float* srow, float m,
                                                 int n, float x) {
  const int lane = threadIdx.x & 31;
  float a = 0.f;
  if (in_regs) {
#pragma unroll
    for (int k = 0; k < kToppPer; ++k) a += e[k] > x ? e[k] : 0.f;
  } else {
    for (int j = lane; j < n; j += 32) {
      const float v = exp2f((srow[j] - m) * 1.4426950408889634f);
      a += v > x ? v : 0.f;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
  return a;
}

__global__ void __launch_bounds__(256) topp_select_kernel(const ToppParams p) {
  extern __shared__ int topp_tab[];
  const int S = p.seq.num_seqs;
  int* s_cu = topp_tab;
  int* s_cb = s_cu + (S + 1);
  int* s_pb = s_cb + (S + 1);
  int* s_ckb = s_pb + (S + 1);
  int* s_ok = s_ckb + (S + 1);
  long long* s_ib = reinterpret_cast<long long*>(((uintptr_t)(s_ok + 1) + 7) & ~(uintptr_t)7);
  if (!build_seq_tables(p.seq, s_cu, s_cb, nullptr, s_ib, p.hq, 0, 0, s_ok, p.dev_status, s_pb, s_ckb)) return;
  if (s_ib[S] != p.index_elems) {
    if (blockIdx.x == 0 && threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
    return;
  }
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const long long rows = (long long)p.hq * p.seq.total_blocks;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows; w += warps) {
    const int h = (int)(w / p.seq.total_blocks), gb = (int)(w % p.seq.total_blocks);
    const int s = find_seq(s_cb, S, gb);
    const int i = gb - s_cb[s];
    const int jd = s_pb[s] + i, n = jd + 1;
    const int64_t base = list_row(s_cb, s_ib, s_pb, s, h, i);
    const float* srow = p.scores + base;
    const bool in_regs = n <= 32 * kToppPer;
    float m = -INFINITY;
    for (int j = lane; j < n; j += 32) m = fmaxf(m, srow[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float e[kToppPer];
    float z = 0.f;
#pragma unroll
    for (int k = 0; k < kToppPer; ++k) {
      const int j = lane + 32 * k;
      e[k] = (in_regs && j < n) ? exp2f((srow[j] - m) * 1.4426950408889634f) : 0.f;
      z += e[k];
    }
    if (!in_regs)
      for (int j = lane; j < n; j += 32) z += exp2f((srow[j] - m) * 1.4426950408889634f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    // the cut x*: keep j iff e_j >= x*  (x* = 0 keeps all, x* above 1 keeps none but the forced)
    uint32_t cut;
    if (p.gamma >= 1.f) {
      cut = 0u;
    } else if (!(p.gamma > 0.f)) {
      cut = 0x7f800000u;  // +inf
    } else {
      const float gz = p.gamma * z;
      uint32_t lo = 0u, hi = 0x3f800000u;  // F(1.0) = 0 < gamma * z
      while (lo < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (topp_mass_above(e, in_regs, srow, m, n, __uint_as_float(mid)) < gz) hi = mid; else lo = mid + 1u;
      }
      cut = lo;
    }
    const float xcut = __uint_as_float(cut);
    int cnt = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      float v = 0.f;
      if (j < n) v = exp2f((srow[j] - m) * 1.4426950408889634f);
      const bool keep = j < n && (j == 0 || j == jd || v >= xcut);
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (keep) p.indices[base + cnt + __popc(bal & lt_mask)] = j;
      cnt += __popc(bal);
    }
    if (lane == 0) p.counts[(long long)h * p.seq.total_blocks + gb] = cnt;
  }
}

cudaError_t launch_topp(const SearchParams& sp, float gamma, float* scores, cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(topp_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)search_smem_bytes(kMaxSeqs));
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cap = 2 * sms;
  const int grid = sp.num_tiles < cap ? sp.num_tiles : cap;
  if (grid <= 0) return cudaSuccess;
  topp_score_kernel<<<grid, kSearchThreads, (int)search_smem_bytes(sp.seq.num_seqs), st>>>(sp, scores);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ToppParams tp;
  tp.seq = sp.seq;
  tp.hq = sp.hq;
  tp.gamma = gamma;
  tp.scores = scores;
  tp.counts = sp.counts;
  tp.indices = sp.indices;
  tp.index_elems = sp.index_elems;
  tp.dev_status = sp.dev_status;
  const size_t tab = (size_t)(4 * (sp.seq.num_seqs + 1) + 1) * 4 + 8 + (size_t)(sp.seq.num_seqs + 1) * 8;
  topp_select_kernel<<<sms * 8, 256, tab, st>>>(tp);
  return cudaGetLastError();
}

// -------------------------------------------------------------------------------- validate ----
// One warp per list row (s, h, i), with jd = pb + i the row's diagonal key block: count in
// [1, jd+1]; entries ascending, in [0, jd]; first 0; last jd.
__global__ void __launch_bounds__(256) validate_kernel(const ValidateParams p) {
  __shared__ int s_cu[kMaxSeqs + 1], s_cb[kMaxSeqs + 1], s_pb[kMaxSeqs + 1], s_ckb[kMaxSeqs + 1];
  __shared__ long long s_ib[kMaxSeqs + 1];
  __shared__ int s_ok;
  if (!build_seq_tables(p.seq, s_cu, s_cb, nullptr, s_ib, p.hq, 0, 0, &s_ok, p.dev_status, s_pb, s_ckb)) return;
  if (s_ib[p.seq.num_seqs] != p.index_elems) {
    if (blockIdx.x == 0 && threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
    return;
  }
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)p.hq * p.seq.total_blocks;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < rows; w += warps) {
    const int h = (int)(w / p.seq.total_blocks), gb = (int)(w % p.seq.total_blocks);
    const int s = find_seq(s_cb, p.seq.num_seqs, gb);
    const int i = gb - s_cb[s];
    const int jd = s_pb[s] + i;
    const int n = p.counts[(long long)h * p.seq.total_blocks + gb];
    bool bad = (n < 1 || n > jd + 1);
    if (!bad) {
      const int32_t* row = p.indices + list_row(s_cb, s_ib, s_pb, s, h, i);
      for (int e = lane; e < n; e += 32) {
        const int x = row[e];
        const int prev = e > 0 ? row[e - 1] : -1;
        if (x < 0 || x > jd || x <= prev) bad = true;
        if (e == 0 && x != 0) bad = true;
        if (e == n - 1 && x != jd) bad = true;
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) dev_flag(p.dev_status, kDevBadList);
  }
}

cudaError_t launch_validate(const ValidateParams& p, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  validate_kernel<<<sms * 4, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace fp
