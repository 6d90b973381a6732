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

// --------------------------------------------------------------- fp32 pooled-score tiles ----
// The exact fp32 pooled scores of a tile (used by the top-p comparison selector, which needs every
// score of a row): CTA tile = (sequence s, kv-head g, TI consecutive query blocks) -> 64 rows
// (q-head, block) that share the pooled keys of kv-head g; pooled keys stream through shared memory
// in chunks of 64 blocks (cp.async, next chunk in flight); warp w scores key blocks 8w..8w+7 of a
// chunk against rows 2l, 2l+1 of lane l (pooled queries transposed in shared memory).
constexpr int kSearchThreads = 256;
constexpr int kSearchRows = 64;
constexpr int kKChunk = 64;                  // key blocks per chunk (8 per warp)
constexpr int kQTStride = kSearchRows + 4;   // transposed pooled-query row stride (floats)
constexpr int kKStride = kHeadDim + 4;       // pooled-key row stride (floats), 16-byte aligned

// Shared memory: fixed part, then the sequence tables sized for this launch's sequence count.
struct SearchSmem {
  float k[2][kKChunk][kKStride];             // pooled keys, natural layout, two buffers
  float qT[kHeadDim][kQTStride];             // pooled queries, [d][row]
  int ok;
};

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

// ---------------------------------------------------------------------------------- search ----
// CTA tile = (sequence s, kv-head g, TI = 128 / G consecutive query blocks) -> up to 128 rows
// (query block i, q-head h) that all read the pooled keys of kv-head g (GQA); row r is block
// i0 + r / G of q-head g*G + r % G and owns TMEM lane r. One persistent CTA per SM, 9 warps:
//   warps 0-3  rows: thread r splits its pooled query into bf16 hi + lo (q = qh + ql + O(2^-16 q))
//              and stores both into TMEM; it reads its row of every score chunk from TMEM;
//   warps 4-7  converters: thread t splits pooled key j0 + t of each 128-key chunk into bf16 hi + lo
//              128-byte-swizzled K-major tiles in shared memory, and tracks the largest |k|;
//   warp 8     allocates TMEM and issues the tcgen05 MMAs from one thread:
//              acc = qh.kh + qh.kl + ql.kh (A from TMEM, B from shared memory, fp32 accumulate),
//              so acc = qbar . kbar = sqrt(d) * s_ij up to |err| <= eps = 2^-13 |qbar| max_j |kbar_j|
//              (the dropped products are below 2^-14.4 sum_d |q_d k_d| and the fp32 accumulation of
//              the 384 products below 2^-17 of it in any order the tensor core may take; both sums
//              are at most |q| |k|, so eps holds with a factor 2 to spare).
// Score chunks flow through a two-stage pipeline: while the rows read chunk c from TMEM, the MMAs
// of chunk c+1 run and the converters fill the shared buffer of chunk c+2.
// Pass A: per row, max and min of acc over the row's causal keys (j <= i). The threshold test
// s_ij - max_j s_ij >= ln(tau) reads acc_j >= max acc + sqrt(d) ln(tau) in these units, and
// |(acc_j - max acc) - sqrt(d) (s_ij - max_j s_ij)| <= 2 eps. A row with (min - max) - 2 eps >=
// sqrt(d) ln(tau) keeps every causal block for certain; a tile whose rows all do is written as
// 0..i and skips pass B.
// Pass B: recompute the chunks and keep block j iff acc_j >= max acc + sqrt(d) ln(tau) (plus the
// sink j = 0 and the diagonal). When 2 eps / sqrt(d) <= 0.99e-4 this decision can differ from the
// exact one only for blocks with |s_ij - max_j s_ij - ln(tau)| < 2 eps / sqrt(d), i.e. inside the
// tie band |p_ij / max p - tau| <= 1e-4 tau, where either decision is correct (the method's own
// tolerance); the rows obey it exactly everywhere else. Kept blocks become per-row keep masks,
// emitted in ascending order by the row's warp with coalesced stores.
// A row whose bound is wider than that (pooled vectors of very large norm; none in the synthetic
// workloads) takes an exact fp32 pass instead: its warp computes every score in fp32, the row max,
// and writes the list in place.
constexpr int kSrchThreads = 288;
constexpr int kSrchRows = 128;                      // rows per tile = TMEM lanes
constexpr int kSrchKeys = 128;                      // pooled keys per chunk = MMA N = TMEM columns per score buffer
constexpr uint32_t kSrchTmemCols = 512;             // S0 | S1 | Qhi | Qlo (384 columns used)
constexpr uint32_t kTmS0 = 0, kTmQh = 256, kTmQl = 320;
constexpr uint32_t kKSlab = kSrchKeys * 128;        // one 64-dim slab of a bf16 key tile (128-byte rows)
constexpr uint32_t kKTile = 2 * kKSlab;             // bf16 key tile (128 dims)
constexpr uint32_t kKBuf = 2 * kKTile;              // hi tile | lo tile
constexpr float kEpsFactor = 1.0f / 8192.0f;        // 2^-13
constexpr float kBandHalf = 0.99e-4f;               // below the tie band's half width in ln units
constexpr uint32_t kIdescSearch = idesc_bf16_f32(128, kSrchKeys, 0, 0);

struct SrchSmem {                  // placed at a 1024-byte aligned address
  unsigned char k[2][kKBuf];       // key chunk buffers
  float kstage[kSrchKeys][kHeadDim];  // fp32 pooled keys of the next chunk to convert (cp.async)
  uint64_t bar_s[2];               // the MMAs of the chunk in buffer b have completed
  uint64_t bar_drain;              // every MMA issued so far has completed (before TMEM is freed)
  uint32_t tmem_base;
  int kmax2_bits;                  // max |kbar_j|^2 over the tile's keys (float bits; >= 0 so int order)
  int need_b;                      // some row of the tile needs pass B
  int need_exact;                  // some row of the tile needs the exact pass
  int ok;
};
// Pooled-query staging at the start of a tile (in the key buffers, free then): 128 rows of 132 floats
constexpr int kQStageStride = kHeadDim + 4;
static_assert(kSrchRows * kQStageStride * 4 <= 2 * kKBuf, "query staging fits in the key buffers");

__host__ __device__ inline size_t srch_smem_bytes(int num_seqs) {
  return sizeof(SrchSmem) + 1024 + (size_t)(num_seqs + 1) * (5 * sizeof(int)) + 8 + (size_t)(num_seqs + 1) * 8;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Exact fp32 dot product of two pooled rows (fixed summation order).
__device__ __forceinline__ float dot128(const float* a, const float* b) {
  float s = 0.f;
#pragma unroll 4
  for (int d = 0; d < kHeadDim; d += 4) {
    const float4 x = *reinterpret_cast<const float4*>(a + d);
    const float4 y = *reinterpret_cast<const float4*>(b + d);
    s = fmaf(x.x, y.x, s);
    s = fmaf(x.y, y.y, s);
    s = fmaf(x.z, y.z, s);
    s = fmaf(x.w, y.w, s);
  }
  return s;
}

// Shared-space accesses of the converters (the role functions below are not inlined, so generic
// pointers would not be known to point at shared memory).
__device__ __forceinline__ float4 lds_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u2(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void cp_async16_s(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes -> 16 zero bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}

// The role code of the search kernel, one copy each (not inlined): the kernel's 9 warps run three
// different instruction streams, and a small hot footprint keeps them in the instruction cache.

// Key split (optional scratch, one launch before the search kernel): every pooled key row (key block
// kb, kv-head g) once, as bf16 hi + lo of its 128 dims (the same split the converters make) and its
// |kbar|^2; one warp per row, lane l holding dims 4l .. 4l + 3.
__global__ void __launch_bounds__(256) ksplit_kernel(const float* __restrict__ k_pool, int64_t rows,
                                                     unsigned char* __restrict__ ksplit, float* __restrict__ knorm2) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += nwarps) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(k_pool + row * kHeadDim) + lane);
    const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
    const uint32_t l01 = pack_bf16x2(v.x - __uint_as_float(h01 << 16), v.y - __uint_as_float(h01 & 0xffff0000u));
    const uint32_t l23 = pack_bf16x2(v.z - __uint_as_float(h23 << 16), v.w - __uint_as_float(h23 & 0xffff0000u));
    unsigned char* dst = ksplit + row * kKeySplitRow + 8 * lane;
    *reinterpret_cast<uint2*>(dst) = make_uint2(h01, h23);
    *reinterpret_cast<uint2*>(dst + 256) = make_uint2(l01, l23);
    // |kbar|^2 in the converters' order: per lane fma chain, then the lane sums of 4-lane groups, then
    // the 8 group sums as a butterfly (the same value on every lane)
    float n2 = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, v.w * v.w)));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
    if (lane == 0) knorm2[row] = n2;
  }
}

// Converters, with a key split: copy the split rows of chunk cc straight into the swizzled key tiles at
// kbuf (lane l < 16: 16 bytes of hi, dims 8l .. 8l + 7; lane l >= 16: the same of lo), zeros past the
// tile's last causal key. Returns the largest |kbar|^2 of the chunk's valid keys this lane read.
__device__ __noinline__ float srch_copy_split(uint32_t kbuf, const unsigned char* ksplit, const float* knorm2, int hkv,
                                              int g, int kb0, int jmax, int cc) {
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - 4;
  const uint32_t piece = lane & 15;
  const uint32_t dst0 = kbuf + ((lane >> 4) ? kKTile : 0u) + (piece >> 3) * kKSlab;
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    const int jr = cw + 4 * i;
    const int j = cc * kSrchKeys + jr;
    const bool valid = j <= jmax;
    const long long row = (long long)(kb0 + (valid ? j : 0)) * hkv + g;
    cp_async16_s(dst0 + jr * 128 + (((piece & 7) ^ (uint32_t)(jr & 7)) << 4), ksplit + row * kKeySplitRow + 16 * lane,
                 valid);
  }
  cp_async_commit();
  const int j = cc * kSrchKeys + cw + 4 * lane;  // lane l reads the norm of key row cw + 4 l
  return j <= jmax ? __ldg(knorm2 + (long long)(kb0 + j) * hkv + g) : 0.f;
}

// Converters: copy this thread's share of the fp32 pooled keys of chunk cc into the staging area:
// converter warp cw takes keys cw, cw + 4, ..., lane l the 16 bytes at dims 4l..4l+3 of each
// (coalesced). A thread later converts exactly the bytes it copied.
__device__ __noinline__ void srch_stage(uint32_t kstage, const float* k_pool, int hkv, int g, int kb0, int jmax,
                                        int cc) {
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - 4;
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    const int jr = cw + 4 * i;
    const int j = cc * kSrchKeys + jr;
    const bool valid = j <= jmax;
    cp_async16_s(kstage + (jr * kHeadDim + 4 * lane) * 4,
                 k_pool + ((long long)(kb0 + (valid ? j : 0)) * hkv + g) * kHeadDim + 4 * lane, valid);
  }
  cp_async_commit();
}

// Converters: split the staged chunk into the bf16 hi + lo tiles at kbuf (128-byte swizzle: the
// 16-byte chunk (l % 16) / 2 of slab row jr sits at chunk ((l % 16) / 2) ^ (jr % 8)). Returns the
// largest |kbar|^2 among the keys whose total this lane ends up holding.
__device__ __noinline__ float srch_convert(uint32_t kstage, uint32_t kbuf) {
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - 4;
  const uint32_t slab_off = (lane >> 4) * kKSlab + ((lane & 1) << 3);
  const uint32_t chunk16 = (lane & 15) >> 1;
  float kmax2 = 0.f;
  cp_async_wait_all();
#pragma unroll 1
  for (int i0b = 0; i0b < 32; i0b += 8) {
    float ps[8];  // this lane's share of |kbar|^2 of each of the batch's 8 keys
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t jr = cw + 4 * (i0b + u);
      const float4 v = lds_f4(kstage + (jr * kHeadDim + 4 * lane) * 4);
      ps[u] = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, v.w * v.w)));
      const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
      const uint32_t l01 = pack_bf16x2(v.x - __uint_as_float(h01 << 16), v.y - __uint_as_float(h01 & 0xffff0000u));
      const uint32_t l23 = pack_bf16x2(v.z - __uint_as_float(h23 << 16), v.w - __uint_as_float(h23 & 0xffff0000u));
      const uint32_t off = slab_off + jr * 128 + ((chunk16 ^ (jr & 7u)) << 4);
      sts_u2(kbuf + off, h01, h23);
      sts_u2(kbuf + kKTile + off, l01, l23);
    }
    // transpose-reduce over the 32 lanes: three halving exchanges leave each lane one key's partial
    // sum over 4 lanes, two butterflies finish it
#pragma unroll
    for (int sft = 16, nv = 4; sft >= 4; sft >>= 1, nv >>= 1) {
      const bool upper = (lane & sft) != 0;
#pragma unroll
      for (int i = 0; i < nv; ++i) {
        const float send = upper ? ps[i] : ps[i + nv];
        const float keep = upper ? ps[i + nv] : ps[i];
        ps[i] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
      }
    }
    ps[0] += __shfl_xor_sync(0xffffffffu, ps[0], 2);
    ps[0] += __shfl_xor_sync(0xffffffffu, ps[0], 1);
    kmax2 = fmaxf(kmax2, ps[0]);
  }
  return kmax2;
}

// MMA thread: acc (TMEM columns d .. d+127) = qh.kh + qh.kl + ql.kh for the key tiles at kbuf.
__device__ __noinline__ void srch_issue(uint32_t tmem, uint32_t d, uint32_t kbuf, uint32_t bar) {
  const uint32_t kh = kbuf, kl = kbuf + kKTile;
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a = tmem + (part == 2 ? kTmQl : kTmQh);
    const uint32_t bb = part == 1 ? kl : kh;
#pragma unroll
    for (int kk = 0; kk < kHeadDim / 16; ++kk) {
      const uint64_t bdesc = sdesc_sw128(bb + (kk >> 2) * kKSlab + (kk & 3) * 32, 16, 1024);
      mma_ts(tmem + d, a + 8 * kk, bdesc, kIdescSearch, (part > 0 || kk > 0) ? 1u : 0u);
    }
  }
  mma_commit(bar);
}

// Rows, pass A: max and min of acc over this row's causal keys of the chunk at TMEM address scol
// (keys j0 .. j0 + 127; the row's last causal key is jd).
__device__ __noinline__ float2 srch_pass_a(uint32_t scol, int j0, int jd, float mx, float mn) {
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    uint32_t a[32];
    tmem_ld32(scol + 32 * q, a);
    tmem_wait_ld();
    reg_fence32(a);
    const int jq = j0 + 32 * q;
    if (jq + 31 <= jd) {
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        mx = fmax3(mx, __uint_as_float(a[e]), __uint_as_float(a[e + 1]));
        mn = fmin3(mn, __uint_as_float(a[e]), __uint_as_float(a[e + 1]));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (jq + e <= jd) {
          mx = fmaxf(mx, __uint_as_float(a[e]));
          mn = fminf(mn, __uint_as_float(a[e]));
        }
    }
  }
  return make_float2(mx, mn);
}

// Rows, pass B: this row's keep mask of the chunk (acc >= thr, the sink, the diagonal, causal keys
// only); then the warp writes the kept blocks of those of its 32 rows that have any in this chunk,
// one row after another, with one coalesced store per 32 keys (the row's masks and list position
// come from its lane by shuffles). rbase / row_n: this thread's row's list start and its blocks kept
// so far; returns the new count.
__device__ __noinline__ int srch_pass_b(uint32_t scol, int j0, int jd, float thr, bool emit, long long rbase,
                                        int row_n, int32_t* indices) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {  // two 32-key loads in flight per wait
    uint32_t a[2][32];
    tmem_ld32(scol + 64 * h, a[0]);  // warp-collective: every lane takes part
    tmem_ld32(scol + 64 * h + 32, a[1]);
    tmem_wait_ld();
    reg_fence32(a[0]);
    reg_fence32(a[1]);
#pragma unroll
    for (int qq = 0; qq < 2; ++qq) {
      uint32_t m = 0u;
#pragma unroll
      for (int e = 0; e < 32; ++e) m |= (__uint_as_float(a[qq][e]) >= thr ? 1u : 0u) << e;
      w[2 * h + qq] = emit ? m : 0u;
    }
  }
  if (emit) {
    if (j0 == 0) w[0] |= 1u;                                                                // the sink
    if (jd >= j0 && jd < j0 + kSrchKeys) w[(jd - j0) >> 5] |= 1u << ((jd - j0) & 31);      // the diagonal
    const int lim = jd - j0 + 1;  // keys j0 .. j0 + lim - 1 are causal
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = lim - 32 * q;
      if (n <= 0) w[q] = 0u;
      else if (n < 32) w[q] &= (1u << n) - 1u;
    }
  }
  const long long mine = rbase + row_n;
  unsigned todo = __ballot_sync(0xffffffffu, (w[0] | w[1] | w[2] | w[3]) != 0u);
  while (todo) {
    const int rr = __ffs(todo) - 1;
    todo &= todo - 1;
    const long long b = (long long)(((unsigned long long)__shfl_sync(0xffffffffu, (unsigned)(mine >> 32), rr) << 32) |
                                    (unsigned)__shfl_sync(0xffffffffu, (unsigned)mine, rr));
    int n = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t m = __shfl_sync(0xffffffffu, w[q], rr);
      if ((m >> lane) & 1u) indices[b + n + __popc(m & lt_mask)] = j0 + 32 * q + lane;
      n += __popc(m);
    }
  }
  return row_n + __popc(w[0]) + __popc(w[1]) + __popc(w[2]) + __popc(w[3]);
}

// Rows of a tile that keeps every causal block: the warp writes 0..jd of each such row of its 32.
__device__ __noinline__ void srch_write_all(bool mine, long long base, int jd, int32_t* indices, int32_t* count) {
  const int lane = threadIdx.x & 31;
  unsigned todo = __ballot_sync(0xffffffffu, mine);
  while (todo) {
    const int rr = __ffs(todo) - 1;
    todo &= todo - 1;
    const long long b = __shfl_sync(0xffffffffu, base, rr);
    const int n = __shfl_sync(0xffffffffu, jd, rr) + 1;
    for (int j = lane; j < n; j += 32) indices[b + j] = j;
  }
  if (mine) *count = jd + 1;
}

// Exact fp32 pass for rows whose bound is wider than the tie band: the row's warp scores every causal
// key with fp32 FMAs (the scores go to the row's own list as scratch), takes the max and compacts the
// kept blocks in place (the writes never pass the entries still to be read).
__device__ __noinline__ void srch_exact_rows(bool mine, long long base, int jd, const float* qrow, const float* k_pool,
                                             int kb0, int hkv, int g, float inv_sqrt_d, float log_tau,
                                             int32_t* indices, int32_t* count) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  unsigned todo = __ballot_sync(0xffffffffu, mine);
  while (todo) {
    const int rr = __ffs(todo) - 1;
    todo &= todo - 1;
    const long long b = __shfl_sync(0xffffffffu, base, rr);
    const int d = __shfl_sync(0xffffffffu, jd, rr);
    const float* qr = reinterpret_cast<const float*>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(qrow), rr));
    float m = -INFINITY;
    for (int j = lane; j <= d; j += 32) {
      const float sc = dot128(qr, k_pool + ((long long)(kb0 + j) * hkv + g) * kHeadDim) * inv_sqrt_d;
      indices[b + j] = __float_as_int(sc);
      m = fmaxf(m, sc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __syncwarp();
    int n = 0;
    for (int jj = 0; jj <= d; jj += 32) {
      const int j = jj + lane;
      const float sc = j <= d ? __int_as_float(indices[b + j]) : -INFINITY;
      __syncwarp();
      const bool keep = j <= d && (j == 0 || j == d || sc - m >= log_tau);
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (keep) indices[b + n + __popc(bal & lt_mask)] = j;
      n += __popc(bal);
      __syncwarp();
    }
    if (lane == rr) *count = n;
  }
}

__global__ void __launch_bounds__(kSrchThreads, 1) search_kernel(const SearchParams p) {
  extern __shared__ __align__(1024) unsigned char srch_raw[];
  SrchSmem& sm = *reinterpret_cast<SrchSmem*>(((uintptr_t)srch_raw + 1023) & ~(uintptr_t)1023);
  const int S = p.seq.num_seqs;
  int* t_cu = reinterpret_cast<int*>(reinterpret_cast<unsigned char*>(&sm) + sizeof(SrchSmem));
  int* t_cb = t_cu + (S + 1);
  int* t_ct = t_cb + (S + 1);
  int* t_pb = t_ct + (S + 1);
  int* t_ckb = t_pb + (S + 1);
  long long* t_ib = reinterpret_cast<long long*>(((uintptr_t)(t_ckb + (S + 1)) + 7) & ~(uintptr_t)7);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool is_row = warp < 4, is_conv = warp >= 4 && warp < 8, is_mma = warp == 8;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.bar_s[0]), 1);
    mbar_init(smem_u32(&sm.bar_s[1]), 1);
    mbar_init(smem_u32(&sm.bar_drain), 1);
    fence_mbar_init();
  }
  if (is_mma) {
    tmem_alloc(smem_u32(&sm.tmem_base), kSrchTmemCols);
    tmem_relinquish();
  }
  const bool ok = build_seq_tables(p.seq, t_cu, t_cb, t_ct, t_ib, p.hq, p.rows_blocks * p.seq.block, p.hkv, &sm.ok,
                                   p.dev_status, t_pb, t_ckb) &&
                  t_ib[S] == p.index_elems;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (!ok && blockIdx.x == 0 && threadIdx.x == 0) dev_flag(p.dev_status, kDevBadProblem);
  const int num_tiles = ok ? t_ct[S] : 0;

  const int G = p.group, TI = p.rows_blocks, NB = p.seq.total_blocks;
  const float sqrt_d = 1.0f / p.inv_sqrt_d;
  const float c_tau = p.log_tau * sqrt_d;            // ln(tau) in acc units (-inf: keep all)
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const uint32_t kstage = smem_u32(&sm.kstage[0][0]);
  const uint32_t kbuf0 = smem_u32(sm.k[0]), kbuf1 = smem_u32(sm.k[1]);
  const uint32_t bar0 = smem_u32(&sm.bar_s[0]), bar1 = smem_u32(&sm.bar_s[1]);
  uint32_t uses0 = 0u, uses1 = 0u;                   // completions of bar_s[0] / bar_s[1] waited on so far
  bool fail = false;

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
    const int jmax = pb + i_last;
    const int nch = jmax / kSrchKeys + 1;

    // ---- this thread's row (rows warps): query block, head, diagonal key block, list start
    const int r = threadIdx.x;
    const bool rvalid = is_row && r < TI * G && i0 + r / G <= i_last;
    const int ri = i0 + r / G, rh = g * G + r % G, rjd = pb + ri;
    const long long rbase = rvalid ? list_row(t_cb, t_ib, t_pb, s, rh, ri) : 0;
    int32_t* rcount = p.counts + (long long)rh * NB + gb0 + ri;
    float qn2 = 0.f;
    if (threadIdx.x == 0) {
      sm.kmax2_bits = 0;
      sm.need_b = 0;
      sm.need_exact = 0;
    }
    int row_n = 0;  // pass B: this row's kept blocks so far
    if (is_row && !p.keep_all) {
      // the pooled queries of this warp's 32 rows: coalesced row copies into the staging area, then
      // each thread splits its own row into bf16 hi + lo and stores both into TMEM (the A operand of
      // the MMAs)
      const uint32_t stage = kbuf0;
#pragma unroll 8
      for (int rr = 0; rr < 32; ++rr) {
        const int r2 = 32 * warp + rr;
        const bool v2 = r2 < TI * G && i0 + r2 / G <= i_last;
        const float* src = p.q_pool + ((long long)(gb0 + i0 + (v2 ? r2 / G : 0)) * p.hq + g * G + r2 % G) * kHeadDim;
        cp_async16_s(stage + (r2 * kQStageStride + 4 * lane) * 4, src + 4 * lane, v2);
      }
      cp_async_commit();
      cp_async_wait_all();
      __syncwarp();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t wh[32], wl[32];
#pragma unroll
        for (int f = 0; f < 16; ++f) {
          const float4 v = lds_f4(stage + (r * kQStageStride + 64 * half + 4 * f) * 4);
          qn2 = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, qn2))));
          const uint32_t h01 = pack_bf16x2(v.x, v.y), h23 = pack_bf16x2(v.z, v.w);
          wh[2 * f] = h01;
          wh[2 * f + 1] = h23;
          wl[2 * f] = pack_bf16x2(v.x - __uint_as_float(h01 << 16), v.y - __uint_as_float(h01 & 0xffff0000u));
          wl[2 * f + 1] = pack_bf16x2(v.z - __uint_as_float(h23 << 16), v.w - __uint_as_float(h23 & 0xffff0000u));
        }
        tmem_st32(tmem + lane_off + kTmQh + 32 * half, wh);
        tmem_st32(tmem + lane_off + kTmQl + 32 * half, wl);
      }
      tmem_wait_st();
      tc_fence_before();
    }
    __syncthreads();  // the staging area becomes the key buffers again
    float mx = -INFINITY, mn = INFINITY;  // pass A: max / min of acc over the row's causal keys
    float kmax2 = 0.f;                    // converters: largest |kbar|^2 seen
    bool keep_all_row = true, exact_row = false, need_b = false;
    float thr = 0.f;

    // ---- pass A (0), then pass B (1) when some row needs it: the same chunk pipeline; while the
    // rows read chunk c from TMEM, the MMAs of chunk c + 1 run and the converters fill chunk c + 2
    for (int pass = p.keep_all ? 2 : 0; pass < 2; ++pass) {
      if (pass == 1 && !need_b) break;
      if (is_conv) {
        if (p.ksplit) {  // split keys: chunks 0 and 1 copied straight into the two key buffers
          kmax2 = fmaxf(kmax2, srch_copy_split(kbuf0, p.ksplit, p.knorm2, p.hkv, g, kb0, jmax, 0));
          if (nch > 1) kmax2 = fmaxf(kmax2, srch_copy_split(kbuf1, p.ksplit, p.knorm2, p.hkv, g, kb0, jmax, 1));
          cp_async_wait_all();
        } else {
          srch_stage(kstage, p.k_pool, p.hkv, g, kb0, jmax, 0);
          kmax2 = fmaxf(kmax2, srch_convert(kstage, kbuf0));
          if (nch > 1) {
            srch_stage(kstage, p.k_pool, p.hkv, g, kb0, jmax, 1);
            kmax2 = fmaxf(kmax2, srch_convert(kstage, kbuf1));
          }
          if (nch > 2) srch_stage(kstage, p.k_pool, p.hkv, g, kb0, jmax, 2);  // lands while the first chunks are scored
        }
        fence_proxy_async_smem();
      }
      __syncthreads();
      if (is_mma && lane == 0) {
        tc_fence_after();
        srch_issue(tmem, kTmS0, kbuf0, bar0);
      }
      for (int c = 0; c < nch; ++c) {
        const int b = c & 1;
        if (is_mma && lane == 0 && c + 1 < nch) srch_issue(tmem, kTmS0 + 128u * (b ^ 1), b ? kbuf0 : kbuf1, b ? bar0 : bar1);
        if (is_row || is_conv) {
          const bool rows = is_row;
          if (rows || c + 2 < nch) {
            // the MMAs of chunk c are done: its scores are in TMEM and buffer b is free again
            const bool done = mbar_wait(b ? bar1 : bar0, (b ? uses1 : uses0) & 1u, p.wait_limit_ns);
            if (rows ? !__all_sync(0xffffffffu, done) : !done) fail = true;
          }
          if (b) ++uses1; else ++uses0;
        }
        if (is_row) {
          tc_fence_after();
          const uint32_t scol = tmem + lane_off + kTmS0 + 128u * b;
          if (pass == 0) {
            const float2 v = srch_pass_a(scol, c * kSrchKeys, rjd, mx, mn);
            mx = v.x;
            mn = v.y;
          } else {
            row_n = srch_pass_b(scol, c * kSrchKeys, rjd, thr, rvalid && !exact_row, rbase, row_n, p.indices);
          }
          tc_fence_before();
        }
        if (is_conv && c + 2 < nch) {
          if (p.ksplit) {  // chunk c + 2 into the buffer that chunk c's MMAs have released
            kmax2 = fmaxf(kmax2, srch_copy_split(b ? kbuf1 : kbuf0, p.ksplit, p.knorm2, p.hkv, g, kb0, jmax, c + 2));
            cp_async_wait_all();
          } else {
            kmax2 = fmaxf(kmax2, srch_convert(kstage, b ? kbuf1 : kbuf0));  // chunk c + 2, staged during chunk c + 1
            if (c + 3 < nch) srch_stage(kstage, p.k_pool, p.hkv, g, kb0, jmax, c + 3);
          }
          fence_proxy_async_smem();
        }
        __syncthreads();
      }
      if (pass == 0) {
        // ---- per-row decision after pass A
        if (is_conv) atomicMax(&sm.kmax2_bits, __float_as_int(kmax2));
        __syncthreads();
        if (is_row && rvalid) {
          const float eps = kEpsFactor * sqrtf(qn2) * sqrtf(__int_as_float(sm.kmax2_bits));
          keep_all_row = (mn - mx) - 2.f * eps >= c_tau;
          exact_row = !keep_all_row && 2.f * eps * p.inv_sqrt_d > kBandHalf;
          thr = mx + c_tau;
          if (!keep_all_row && !exact_row) atomicOr(&sm.need_b, 1);
          if (exact_row) atomicOr(&sm.need_exact, 1);
        }
        __syncthreads();
        need_b = sm.need_b != 0;
      }
    }

    if (is_row) {
      if (!need_b) {
        // every row keeps all of its causal blocks (or needs the exact pass): write 0..i
        srch_write_all(rvalid && keep_all_row, rbase, rjd, p.indices, rcount);
      } else if (rvalid && !exact_row) {
        *rcount = row_n;
      }
      if (sm.need_exact)
        srch_exact_rows(rvalid && exact_row, rbase, rjd, p.q_pool + ((long long)(gb0 + ri) * p.hq + rh) * kHeadDim,
                        p.k_pool, kb0, p.hkv, g, p.inv_sqrt_d, p.log_tau, p.indices, rcount);
    }
    __syncthreads();  // the next tile reuses TMEM, the buffers and the flags
    if (__syncthreads_or(fail)) break;
  }
  if (fail && threadIdx.x == 0) dev_flag(p.dev_status, kDevTimeout);

  if (is_mma) {
    // every issued MMA has completed before TMEM is released (own, generous limit: MMAs always finish)
    if (lane == 0) {
      mma_commit(smem_u32(&sm.bar_drain));
      mbar_wait(smem_u32(&sm.bar_drain), 0, 1000000000ull);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (is_mma) tmem_dealloc(tmem, kSrchTmemCols);
}

cudaError_t launch_search(const SearchParams& sp, cudaStream_t st) {
  static unsigned long long attr_done[kMaxCachedDevices] = {};
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(search_kernel), (int)srch_smem_bytes(kMaxSeqs), attr_done);
  if (e != cudaSuccess) return e;
  SearchParams p = sp;
  p.rows_blocks = kSrchRows / p.group;  // query blocks per tile (G <= 64)
  const long long tiles = (long long)p.hkv * (p.seq.total_blocks / p.rows_blocks + p.seq.num_seqs);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)(tiles < sms ? tiles : sms);
  if (grid <= 0) return cudaSuccess;
  if (p.ksplit) {  // every pooled key split once, before the tiles read them
    const int64_t rows = (int64_t)p.seq.total_kv_blocks * p.hkv;
    const int64_t blocks = (rows + 7) / 8;
    ksplit_kernel<<<(int)(blocks < 8 * sms ? blocks : 8 * sms), 256, 0, st>>>(p.k_pool, rows, p.ksplit, p.knorm2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  search_kernel<<<grid, kSrchThreads, srch_smem_bytes(p.seq.num_seqs), st>>>(p);
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
  static unsigned long long attr_done[kMaxCachedDevices] = {};
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(topp_score_kernel), (int)search_smem_bytes(kMaxSeqs),
                               attr_done);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int cap = 2 * sms;
  const int grid = sp.num_tiles < cap ? sp.num_tiles : cap;
  if (grid <= 0) return cudaSuccess;
  topp_score_kernel<<<grid, kSearchThreads, (int)search_smem_bytes(sp.seq.num_seqs), st>>>(sp, scores);
  e = cudaGetLastError();
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
