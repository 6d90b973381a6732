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

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const PoolParams p) {
  __shared__ int s_cu[kMaxSeqs + 1], s_cb[kMaxSeqs + 1];
  __shared__ int s_ok;
  if (!build_seq_tables(p.seq, s_cu, s_cb, nullptr, nullptr, 0, 0, 0, &s_ok, p.dev_status)) return;
  const int S = p.seq.num_seqs, B = p.seq.block;
  const int per_block = p.q_chunks + p.k_chunks;
  const long long items = (long long)p.seq.total_blocks * per_block;
  for (long long w = blockIdx.x; w < items; w += gridDim.x) {
    const int gb = (int)(w / per_block);
    const int part = (int)(w % per_block);
    const int s = find_seq(s_cb, S, gb);
    const int i = gb - s_cb[s];
    const int t0 = s_cu[s] + i * B;
    const int t1 = min(t0 + B, s_cu[s + 1]);
    const bool is_q = part < p.q_chunks;
    const int row = is_q ? p.q_row : p.k_row;
    const int col = (is_q ? part : part - p.q_chunks) * kPoolChunk + threadIdx.x * 8;
    if (col >= row) continue;
    const uint16_t* src = (is_q ? p.q : p.k) + (long long)t0 * row + col;
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int t = t0;
    for (; t + 8 <= t1; t += 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = ld_stream_16(src + (long long)(t - t0 + u) * row);
#pragma unroll
      for (int u = 0; u < 8; ++u) acc_bf16x8(a, v[u]);
    }
    for (; t < t1; ++t) acc_bf16x8(a, ld_stream_16(src + (long long)(t - t0) * row));
    const float inv_n = 1.0f / (float)(t1 - t0);
    float* dst = (is_q ? p.q_pool : p.k_pool) + (long long)gb * row + col;
    float4 o0 = make_float4(a[0] * inv_n, a[1] * inv_n, a[2] * inv_n, a[3] * inv_n);
    float4 o1 = make_float4(a[4] * inv_n, a[5] * inv_n, a[6] * inv_n, a[7] * inv_n);
    reinterpret_cast<float4*>(dst)[0] = o0;
    reinterpret_cast<float4*>(dst)[1] = o1;
  }
}

cudaError_t launch_pool(const PoolParams& p, int grid, cudaStream_t st) {
  pool_kernel<<<grid, kPoolThreads, 0, st>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------- search ----
// CTA tile = (sequence s, kv-head g, TI consecutive query blocks) -> 64 rows (q-head, block) that
// all share the pooled keys of kv-head g (GQA). Row r: head offset r % G, block offset r / G.
// Pooled keys stream through shared memory in chunks of 64 blocks, double buffered with cp.async
// (16-byte global->shared copies in flight while the previous chunk is scored). Warp w scores key
// blocks 8w..8w+7 of a chunk (broadcast shared reads) against rows 2l, 2l+1 of lane l (pooled
// queries transposed in shared memory): per 4 steps of d, 8 broadcast and 4 lane-private loads
// feed 64 FMAs, so the loop is bound by the FMA pipe.
// Pass 1: row max m_i and row min of s_ij over j <= i (scores stay in registers).
// If min - max >= ln(tau) every causal block passes (fp32 subtraction is monotonic, so this is the
// same decision the per-block test would take) and the row is written as 0..i directly.
// Otherwise pass 2 recomputes the scores, stages them in shared memory, and one warp per 8 rows
// emits the kept blocks in ascending order with ballot/popc compaction.
constexpr int kSearchThreads = 256;
constexpr int kSearchWarps = kSearchThreads / 32;
constexpr int kSearchRows = 64;
constexpr int kKChunk = 64;                  // key blocks per chunk (8 per warp)
constexpr int kQTStride = kSearchRows + 4;   // transposed pooled-query row stride (floats)
constexpr int kKStride = kHeadDim + 4;       // pooled-key row stride (floats), 16-byte aligned

struct SearchSmem {
  float k[2][kKChunk][kKStride];             // pooled keys, natural layout, two buffers
  float qT[kHeadDim][kQTStride];             // pooled queries, [d][row]
  float red[2][kSearchWarps][kSearchRows];   // per-warp row max / min
  float sc[kSearchRows][kKChunk + 1];        // chunk scores for the emission pass
  int cu[kMaxSeqs + 1], cb[kMaxSeqs + 1], ct[kMaxSeqs + 1];
  long long ib[kMaxSeqs + 1];
  int ok;
  int need_pass2;
};

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

__global__ void __launch_bounds__(kSearchThreads, 1) search_kernel(const SearchParams p) {
  extern __shared__ __align__(16) unsigned char search_smem_raw[];
  SearchSmem& sm = *reinterpret_cast<SearchSmem*>(search_smem_raw);
  if (!build_seq_tables(p.seq, sm.cu, sm.cb, sm.ct, sm.ib, p.hq, p.rows_blocks * p.seq.block, p.hkv, &sm.ok,
                        p.dev_status))
    return;
  const int S = p.seq.num_seqs;
  if (sm.ib[S] != p.index_elems) {
    if (blockIdx.x == 0 && threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
    return;
  }
  const int G = p.group, TI = p.rows_blocks;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NB = p.seq.total_blocks;
  const unsigned lt_mask = (1u << lane) - 1u;

  const int num_tiles = sm.ct[S];
  for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
    const int s = find_seq(sm.ct, S, tile);
    const int local = tile - sm.ct[s];
    const int nb = sm.cb[s + 1] - sm.cb[s];
    const int ntiles = (nb + TI - 1) / TI;
    const int it = ntiles - 1 - local / p.hkv;  // heavy (late) query blocks first
    const int g = local % p.hkv;
    const int i0 = it * TI;
    const int i_last = min(i0 + TI, nb) - 1;
    const int gb0 = sm.cb[s];
    const int nchunks = i_last / kKChunk + 1;

    __syncthreads();  // previous tile done with shared memory
    if (!p.keep_all) issue_k_chunk(sm, 0, p.k_pool, gb0, g, p.hkv, 0, i_last);
    for (int e = threadIdx.x; e < kSearchRows * (kHeadDim / 4); e += kSearchThreads) {
      const int r = e % kSearchRows, d4 = e / kSearchRows;
      const int i = i0 + r / G, h = g * G + r % G;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < TI * G && i <= i_last)
        v = reinterpret_cast<const float4*>(p.q_pool + ((long long)(gb0 + i) * p.hq + h) * kHeadDim)[d4];
      sm.qT[4 * d4 + 0][r] = v.x;
      sm.qT[4 * d4 + 1][r] = v.y;
      sm.qT[4 * d4 + 2][r] = v.z;
      sm.qT[4 * d4 + 3][r] = v.w;
    }
    if (threadIdx.x == 0) sm.need_pass2 = 0;

    // scoring rows of this lane
    int li[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 2 * lane + e;
      li[e] = (r < TI * G && i0 + r / G <= i_last) ? i0 + r / G : -1;
    }
    float mx[2] = {-INFINITY, -INFINITY}, mn[2] = {INFINITY, INFINITY};

    if (!p.keep_all) {
      // ---- pass 1: row max / min of the pooled scores
      for (int c = 0; c < nchunks; ++c) {
        const int j0 = c * kKChunk;
        if (c + 1 < nchunks) {
          __syncthreads();  // buffer (c+1)&1 no longer read
          issue_k_chunk(sm, (c + 1) & 1, p.k_pool, gb0, g, p.hkv, j0 + kKChunk, i_last);
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
    }
    __syncthreads();

    // emission rows: warp w emits rows 8w..8w+7
    int row_i[8], row_h[8];
    float rmx[8];
    bool all_keep[8];
    bool warp_needs = false;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int rr = warp * 8 + r;
      row_i[r] = (rr < TI * G && i0 + rr / G <= i_last) ? i0 + rr / G : -1;
      row_h[r] = g * G + rr % G;
      float a = -INFINITY, b = INFINITY;
      if (!p.keep_all) {
#pragma unroll
        for (int w = 0; w < kSearchWarps; ++w) {
          a = fmaxf(a, sm.red[0][w][rr]);
          b = fminf(b, sm.red[1][w][rr]);
        }
      }
      rmx[r] = a;
      all_keep[r] = p.keep_all || (b - a >= p.log_tau);
      if (row_i[r] >= 0 && !all_keep[r]) warp_needs = true;
    }
    const int warp_imax = max(max(max(row_i[0], row_i[1]), max(row_i[2], row_i[3])),
                              max(max(row_i[4], row_i[5]), max(row_i[6], row_i[7])));
    if (warp_needs && lane == 0) atomicOr(&sm.need_pass2, 1);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (row_i[r] < 0 || !all_keep[r]) continue;
      const int i = row_i[r];
      int32_t* dst = p.indices + list_row(sm.cb, sm.ib, s, row_h[r], i);
      for (int j = lane; j <= i; j += 32) dst[j] = j;
      if (lane == 0) p.counts[(long long)row_h[r] * NB + gb0 + i] = i + 1;
    }
    __syncthreads();
    if (!sm.need_pass2) continue;

    // ---- pass 2: recompute the scores and emit kept blocks in ascending order
    int cnt[8];
    int64_t base[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      cnt[r] = 0;
      base[r] = (row_i[r] >= 0) ? list_row(sm.cb, sm.ib, s, row_h[r], row_i[r]) : 0;
    }
    for (int c = 0; c < nchunks; ++c) {
      const int j0 = c * kKChunk;
      __syncthreads();
      issue_k_chunk(sm, 0, p.k_pool, gb0, g, p.hkv, j0, i_last);
      cp_async_wait_all();
      __syncthreads();
      float acc[2][8];
      chunk_scores(sm, 0, warp, lane, acc);
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int b = 0; b < 8; ++b) sm.sc[2 * lane + e][8 * warp + b] = acc[e][b] * p.inv_sqrt_d;
      __syncthreads();
      if (!warp_needs || j0 > warp_imax) continue;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (row_i[r] < 0 || all_keep[r] || j0 > row_i[r]) continue;
#pragma unroll
        for (int h2 = 0; h2 < kKChunk; h2 += 32) {
          const int j = j0 + h2 + lane;
          const float sc = sm.sc[warp * 8 + r][h2 + lane];
          const bool keep = j <= row_i[r] && (j == 0 || j == row_i[r] || sc - rmx[r] >= p.log_tau);
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
  const int smem = (int)sizeof(SearchSmem);
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(search_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.num_tiles < sms ? p.num_tiles : sms;
  if (grid <= 0) return cudaSuccess;
  search_kernel<<<grid, kSearchThreads, smem, st>>>(p);
  return cudaGetLastError();
}

// -------------------------------------------------------------------------------- validate ----
// One warp per list row (s, h, i): count in [1, i+1]; entries ascending, in [0, i]; first 0; last i.
__global__ void __launch_bounds__(256) validate_kernel(const ValidateParams p) {
  __shared__ int s_cu[kMaxSeqs + 1], s_cb[kMaxSeqs + 1];
  __shared__ long long s_ib[kMaxSeqs + 1];
  __shared__ int s_ok;
  if (!build_seq_tables(p.seq, s_cu, s_cb, nullptr, s_ib, p.hq, 0, 0, &s_ok, p.dev_status)) return;
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
    const int n = p.counts[(long long)h * p.seq.total_blocks + gb];
    bool bad = (n < 1 || n > i + 1);
    if (!bad) {
      const int32_t* row = p.indices + list_row(s_cb, s_ib, s, h, i);
      for (int e = lane; e < n; e += 32) {
        const int x = row[e];
        const int prev = e > 0 ? row[e - 1] : -1;
        if (x < 0 || x > i || x <= prev) bad = true;
        if (e == 0 && x != 0) bad = true;
        if (e == n - 1 && x != i) bad = true;
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
