// fp_internal.h -- launch parameter structs and launcher declarations shared by the CUDA sources
// of libfp (not part of the public ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/fp.h"

namespace fp {

struct SeqInfo {
  const int32_t* cu_seqlens;  // device [S+1], the queries (and, without a cache, the keys)
  int32_t num_seqs;
  int32_t total_tokens;
  int32_t total_blocks;       // query blocks
  int32_t block;              // B
  // Chunked prefill onto a key/value cache (all zero / null for a plain prefill): sequence s has
  // prefix_lens[s] cached tokens (a multiple of B) before its L_s queries, so its keys are the
  // prefix_lens[s] + L_s tokens of the cache and its query block i is key block prefix/B + i.
  const int32_t* prefix_lens; // device [S] or null
  int32_t total_kv_blocks;    // sum_s ceil((prefix_s + L_s) / B) (== total_blocks without a cache)
  // Paged cache (block_table null: K/V are [total_tokens, Hkv, d] indexed by cu_seqlens):
  // key token u of sequence s is row block_table[s * max_pages + u / page_size] * page_size +
  // u % page_size of the cache (page_size is a multiple of B, so a key block never straddles pages).
  const int32_t* block_table; // device [S, max_pages] or null
  int32_t max_pages;
  int32_t page_size;
  int32_t num_pages;          // pages in the cache (entries outside [0, num_pages) are rejected)
};

struct PoolParams {
  SeqInfo seq;
  const uint16_t* q;          // [T, Hq, d] bf16 bits
  const uint16_t* k;          // [T, Hkv, d], or the paged cache [pages * page_size, Hkv, d]
  float* q_pool;              // [NB, Hq, d]
  float* k_pool;              // [NBK, Hkv, d] (NBK = seq.total_kv_blocks)
  int32_t q_row;              // Hq * d
  int32_t k_row;              // Hkv * d
  int32_t q_chunks, k_chunks; // 1024-element column chunks per token row
  int32_t* dev_status;
};

struct SearchParams {
  SeqInfo seq;
  const float* q_pool;        // pooled queries [NB, Hq, d]
  const float* k_pool;        // pooled keys [NBK, Hkv, d]
  int32_t hq, hkv, group;     // group = Hq / Hkv
  int32_t rows_blocks;        // query blocks per CTA tile (TI)
  int32_t num_tiles;          // grid-size hint (upper bound); the exact count is s_ct[S] on device
  float inv_sqrt_d;
  float log_tau;              // threshold on s - max (natural log units); -inf keeps all
  int32_t keep_all;           // tau <= 0
  int32_t* counts;            // [Hq, NB]
  int32_t* indices;           // row (s, h, i) at base_s + h*(nb*pb + nb(nb+1)/2) + i*pb + i(i+1)/2
  int64_t index_elems;
  int32_t* dev_status;
  uint64_t wait_limit_ns;     // limit of every bounded wait of the search kernel
  // optional key split (null: each tile splits the keys it reads): row (key block kb, kv-head g) at
  // ksplit + (kb * hkv + g) * kKeySplitRow holds bf16 hi of the 128 dims, then bf16 lo; knorm2 the
  // row's |kbar|^2; both written by the split kernel at the start of the search launch
  unsigned char* ksplit;
  float* knorm2;
};

constexpr int64_t kKeySplitRow = 512;  // bytes per (key block, kv-head): 128 bf16 hi + 128 bf16 lo
// Layout of the key split buffer for nbk key blocks: split rows, then (256-byte aligned) the norms.
struct KeySplitLayout {
  int64_t norms, total;
};
inline KeySplitLayout key_split_layout(int64_t nbk, int64_t hkv) {
  KeySplitLayout l;
  l.norms = (nbk * hkv * kKeySplitRow + 255) & ~(int64_t)255;
  l.total = (l.norms + nbk * hkv * 4 + 255) & ~(int64_t)255;
  return l;
}

struct ValidateParams {
  SeqInfo seq;
  int32_t hq;
  const int32_t* counts;
  const int32_t* indices;
  int64_t index_elems;
  int32_t* dev_status;
};

struct __align__(64) AttnParams {
  CUtensorMap tm_q;           // Q as 2-D [T rows, Hq*d cols], box {64, 128}, 128B swizzle
  CUtensorMap tm_k;           // K as 2-D [T (or pages * page_size) rows, Hkv*d cols], box {64, B}
  CUtensorMap tm_v;           // V likewise
  SeqInfo seq;
  int32_t hq, hkv, group;
  int32_t num_tiles;          // unused by the kernel (exact count is s_ct[S] on device)
  int32_t dense;              // 1: every causal block; 0: counts/indices lists
  const int32_t* counts;
  const int32_t* indices;
  int64_t index_elems;
  float scale_log2;           // softmax_scale * log2(e)
  uint16_t* out;              // [T, Hq, d] bf16 bits
  int32_t out32;              // out is 32-byte aligned: the epilogue stores 32 bytes per instruction
  float* lse;                 // [Hq, T] or null
  int32_t* dev_status;
  uint64_t wait_limit_ns;
  int32_t test_unsignalled_wait;  // test hook: softmax warps first wait on a barrier nothing signals
  int32_t units;                  // attention schedule: 0 by list density, 1 tile pairs, 2 single tiles
  int32_t fp8;                    // 1: tm_q / tm_k are e4m3 (uint8) maps, box {128, rows}; scales folded into scale_log2
  int32_t* sched;                 // work counter (next unit, finished CTAs), zero at launch and exit; or null
  const int8_t* q_exp;            // fp8 with per-block scales: q-block scale 2^q_exp[global block * hq + h], or null
  const int8_t* k_exp;            // and key-block scale 2^k_exp[global block * hkv + g]
};

constexpr int kMaxSeqs = FP_MAX_SEQS;
constexpr int kHeadDim = 128;
constexpr int kTileM = 128;   // query rows per attention tile

// Record the message returned by fp_last_error() and return `st`.
fp_status set_error(fp_status st, const char* fmt, ...);

// Unique id of the calling thread's current CUDA context (cuCtxGetId), 0 when there is none or the
// driver cannot tell. Per-device state that a context owns (function attributes, the device address
// of a static array) is cached under this id, so a context destroyed and created again (for example
// by cudaDeviceReset) is never mistaken for the old one.
unsigned long long context_id();

// cudaFuncSetAttribute(func, MaxDynamicSharedMemorySize, bytes) once per device context: the
// attribute belongs to the current device's context, so `done[dev]` remembers the context id it was
// set in (ordinals >= kMaxCachedDevices set it at every call).
constexpr int kMaxCachedDevices = 64;
cudaError_t set_max_smem(const void* func, int bytes, unsigned long long (&done)[kMaxCachedDevices]);

cudaError_t launch_pool(const PoolParams& p, int grid, cudaStream_t st);
cudaError_t launch_search(const SearchParams& p, cudaStream_t st);
cudaError_t launch_validate(const ValidateParams& p, cudaStream_t st);
// Cumulative top-p selection (comparison selector): scores scratch [index_elems] floats.
cudaError_t launch_topp(const SearchParams& p, float gamma, float* scores, cudaStream_t st);
cudaError_t launch_attn(const AttnParams& p, int grid, cudaStream_t st);
cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_mufu, long long n, cudaStream_t st);

}  // namespace fp
