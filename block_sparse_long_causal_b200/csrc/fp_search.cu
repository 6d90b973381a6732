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
// Warp w owns rows 8w..8w+7 and lane l owns key blocks j0+2l, j0+2l+1 of a 64-block chunk; the
// scores are a register-tiled outer product over d with pooled queries and keys transposed in
// shared memory: per step of d, two broadcast 16-byte loads (8 rows, same for the whole warp) and
// one 8-byte load per lane feed 16 FMAs, so the loop is bound by the FMA pipe, not shared memory.
// Pass 1: row max m_i and row min of s_ij over j <= i (scores stay in registers).
// If min - max >= ln(tau) every causal block passes (fp32 subtraction is monotonic, so this is the
// same decision the per-block test would take) and the row is written as 0..i directly.
// Otherwise pass 2 recomputes the scores and emits kept blocks in ascending order with two ballots
// per row and chunk (even and odd key blocks) and popc prefix counts.
constexpr int kSearchThreads = 256;
constexpr int kSearchRows = 64;
constexpr int kKChunk = 64;
constexpr int kTStride = kSearchRows + 4;  // transposed row stride (floats); 16-byte aligned

struct SearchSmem {
  float qT[kHeadDim][kTStride];   // pooled queries, [d][row]
  float kT[kHeadDim][kTStride];   // pooled keys of the current chunk, [d][j]
  int cu[kMaxSeqs + 1], cb[kMaxSeqs + 1], ct[kMaxSeqs + 1];
  long long ib[kMaxSeqs + 1];
  int ok;
  int need_pass2;
};

// kT[d][jr] = kbar[gb0 + j0 + jr][g][d] (zero past jmax). Lane <-> key block so that the transposed
// shared stores are conflict free; the loads are 16-byte pieces of L2-resident rows.
__device__ __forceinline__ void load_k_chunk(SearchSmem& sm, const float* kp, int gb0, int g, int hkv, int j0,
                                             int jmax) {
  for (int e = threadIdx.x; e < kKChunk * (kHeadDim / 4); e += kSearchThreads) {
    const int jr = e % kKChunk, d4 = e / kKChunk;
    const int j = j0 + jr;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j <= jmax) v = reinterpret_cast<const float4*>(kp + ((long long)(gb0 + j) * hkv + g) * kHeadDim)[d4];
    sm.kT[4 * d4 + 0][jr] = v.x;
    sm.kT[4 * d4 + 1][jr] = v.y;
    sm.kT[4 * d4 + 2][jr] = v.z;
    sm.kT[4 * d4 + 3][jr] = v.w;
  }
}

// acc[r][e] = q_row(8w+r) . k_block(2*lane+e) over the full head dim.
__device__ __forceinline__ void chunk_scores(const SearchSmem& sm, int warp, int lane, float (&acc)[8][2]) {
#pragma unroll
  for (int r = 0; r < 8; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll 8
  for (int d = 0; d < kHeadDim; ++d) {
    const float4 qa = *reinterpret_cast<const float4*>(&sm.qT[d][8 * warp]);
    const float4 qb = *reinterpret_cast<const float4*>(&sm.qT[d][8 * warp + 4]);
    const float2 kv = *reinterpret_cast<const float2*>(&sm.kT[d][2 * lane]);
    const float q8[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      acc[r][0] = fmaf(q8[r], kv.x, acc[r][0]);
      acc[r][1] = fmaf(q8[r], kv.y, acc[r][1]);
    }
  }
}

__global__ void __launch_bounds__(kSearchThreads) search_kernel(const SearchParams p) {
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

    __syncthreads();  // previous tile done with shared memory
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

    int row_i[8], row_h[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int rr = warp * 8 + r;
      row_i[r] = (rr < TI * G && i0 + rr / G <= i_last) ? i0 + rr / G : -1;
      row_h[r] = g * G + rr % G;
    }
    const int warp_imax = max(max(max(row_i[0], row_i[1]), max(row_i[2], row_i[3])),
                              max(max(row_i[4], row_i[5]), max(row_i[6], row_i[7])));
    float mx[8], mn[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) { mx[r] = -INFINITY; mn[r] = INFINITY; }

    if (!p.keep_all) {
      // ---- pass 1: row max / min of the pooled scores
      for (int j0 = 0; j0 <= i_last; j0 += kKChunk) {
        __syncthreads();
        load_k_chunk(sm, p.k_pool, gb0, g, p.hkv, j0, i_last);
        __syncthreads();
        if (j0 > warp_imax) continue;
        float acc[8][2];
        chunk_scores(sm, warp, lane, acc);
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (j0 + 2 * lane + e <= row_i[r]) {
              const float sc = acc[r][e] * p.inv_sqrt_d;
              mx[r] = fmaxf(mx[r], sc);
              mn[r] = fminf(mn[r], sc);
            }
          }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], o));
          mn[r] = fminf(mn[r], __shfl_xor_sync(0xffffffffu, mn[r], o));
        }
      }
    }

    // rows whose every causal block passes are written as 0..i without recomputation
    bool all_keep[8];
    bool warp_needs = false;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      all_keep[r] = p.keep_all || (mn[r] - mx[r] >= p.log_tau);
      if (row_i[r] >= 0 && !all_keep[r]) warp_needs = true;
    }
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
    for (int j0 = 0; j0 <= i_last; j0 += kKChunk) {
      __syncthreads();
      load_k_chunk(sm, p.k_pool, gb0, g, p.hkv, j0, i_last);
      __syncthreads();
      if (!warp_needs || j0 > warp_imax) continue;
      float acc[8][2];
      chunk_scores(sm, warp, lane, acc);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (row_i[r] < 0 || all_keep[r] || j0 > row_i[r]) continue;
        bool keep[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + 2 * lane + e;
          keep[e] = j <= row_i[r] && (j == 0 || j == row_i[r] || acc[r][e] * p.inv_sqrt_d - mx[r] >= p.log_tau);
        }
        const unsigned b0 = __ballot_sync(0xffffffffu, keep[0]);
        const unsigned b1 = __ballot_sync(0xffffffffu, keep[1]);
        // ascending order j0 + 2l + e: entries before (l, e) are both of lanes < l, plus (l, 0) for e = 1
        const int before = cnt[r] + __popc(b0 & lt_mask) + __popc(b1 & lt_mask);
        if (keep[0]) p.indices[base[r] + before] = j0 + 2 * lane;
        if (keep[1]) p.indices[base[r] + before + (keep[0] ? 1 : 0)] = j0 + 2 * lane + 1;
        cnt[r] += __popc(b0) + __popc(b1);
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
  const int grid = p.num_tiles < sms * 4 ? p.num_tiles : sms * 4;
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
