// fp_api.cu -- the extern "C" boundary of libfp: argument checks, TMA tensor maps and launches.
// See include/fp.h for the contract of every entry point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fp_internal.h"

namespace {

thread_local char g_err[512] = "no error";

fp_status fail(fp_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

fp_status check_problem(const fp_problem* p) {
  if (!p) return fail(FP_ERR_INVALID_ARG, "problem is NULL");
  if (!p->cu_seqlens) return fail(FP_ERR_INVALID_ARG, "problem.cu_seqlens is NULL");
  if (p->num_seqs < 1 || p->num_seqs > FP_MAX_SEQS)
    return fail(FP_ERR_INVALID_ARG, "num_seqs=%d outside [1, %d]", p->num_seqs, FP_MAX_SEQS);
  if (p->num_q_heads < 1 || p->num_kv_heads < 1 || p->num_q_heads % p->num_kv_heads)
    return fail(FP_ERR_INVALID_ARG, "num_q_heads=%d must be a positive multiple of num_kv_heads=%d",
                p->num_q_heads, p->num_kv_heads);
  if (p->num_q_heads / p->num_kv_heads > 64)
    return fail(FP_ERR_UNSUPPORTED, "GQA group size %d > 64", p->num_q_heads / p->num_kv_heads);
  if (p->head_dim != 128) return fail(FP_ERR_UNSUPPORTED, "head_dim=%d (only 128 is built)", p->head_dim);
  if (p->block_size != 64 && p->block_size != 128)
    return fail(FP_ERR_UNSUPPORTED, "block_size=%d (64 or 128)", p->block_size);
  if (p->total_tokens < 0 || p->total_blocks < 0 || p->index_elems < 0)
    return fail(FP_ERR_INVALID_ARG, "negative sizes in problem (use fp_problem_init)");
  return FP_OK;
}

fp_status check_cache(const fp_problem* p, const fp_paged_cache* c) {
  if (!c) return FP_OK;
  if (!c->prefix_lens || !c->block_table)
    return fail(FP_ERR_INVALID_ARG, "cache.prefix_lens and cache.block_table must be non-NULL (use fp_paged_cache_init)");
  if (c->page_size <= 0 || c->page_size % p->block_size || c->max_pages < 1 || c->num_pages < 1 ||
      c->total_kv_blocks < p->total_blocks || c->index_elems < p->index_elems)
    return fail(FP_ERR_INVALID_ARG, "inconsistent paged cache (use fp_paged_cache_init)");
  return FP_OK;
}

// c == NULL: a plain prefill (keys = the queries' tokens, K/V indexed by cu_seqlens)
fp::SeqInfo seq_info(const fp_problem* p, const fp_paged_cache* c = nullptr) {
  fp::SeqInfo s;
  memset(&s, 0, sizeof s);
  s.cu_seqlens = p->cu_seqlens;
  s.num_seqs = p->num_seqs;
  s.total_tokens = p->total_tokens;
  s.total_blocks = p->total_blocks;
  s.block = p->block_size;
  s.total_kv_blocks = c ? c->total_kv_blocks : p->total_blocks;
  if (c) {
    s.prefix_lens = c->prefix_lens;
    s.block_table = c->block_table;
    s.max_pages = c->max_pages;
    s.page_size = c->page_size;
    s.num_pages = c->num_pages;
  }
  return s;
}
int64_t index_elems(const fp_problem* p, const fp_paged_cache* c) { return c ? c->index_elems : p->index_elems; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows, cols] row-major, 128-byte swizzle, zero fill out of range. bf16: box {64 cols, box_rows};
// one-byte elements (e4m3 carried as uint8): box {128 cols, box_rows}. Either way a box row is
// one 128-byte swizzle atom.
fp_status make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows, bool byte_elems = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int el = byte_elems ? 1 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)(rows > 0 ? rows : 1)};
  cuuint64_t strides[1] = {(cuuint64_t)cols * el};
  cuuint32_t box[2] = {(cuuint32_t)(128 / el), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(m, byte_elems ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FP_OK;
}

fp_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return FP_OK;
  return fail(FP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Limit of every bounded wait inside the attention kernel: 2 s, or FP_WAIT_LIMIT_MS (read at each
// call, so a test can make the waits run out on purpose).
uint64_t wait_limit_ns() {
  const char* s = getenv("FP_WAIT_LIMIT_MS");
  double ms = s ? atof(s) : 2000.0;
  if (!(ms > 0.0)) ms = 2000.0;
  return (uint64_t)(ms * 1e6) > 0 ? (uint64_t)(ms * 1e6) : 1;
}

// fp8: q and k hold e4m3 codes (one byte per element) and the logits are
// softmax_scale * (qk_scale * q . k), qk_scale = q_scale * k_scale.
fp_status attn_common(const fp_problem* p, const fp_paged_cache* c, const void* q, const void* k, const void* v,
                      const int32_t* counts, const int32_t* indices, int dense, float softmax_scale, void* out,
                      float* lse, int32_t* dev_status, void* stream, bool fp8 = false, float qk_scale = 1.f,
                      const int8_t* q_exp = nullptr, const int8_t* k_exp = nullptr) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if ((st = check_cache(p, c)) != FP_OK) return st;
  if (!q || !k || !v || !out) return fail(FP_ERR_INVALID_ARG, "q, k, v and out must be non-NULL");
  if (!dense && (!counts || !indices)) return fail(FP_ERR_INVALID_ARG, "counts and indices must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(FP_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
  if (!std::isfinite(softmax_scale)) return fail(FP_ERR_INVALID_ARG, "softmax_scale is not finite");
  if ((reinterpret_cast<uintptr_t>(p->sched) & 3u) != 0) return fail(FP_ERR_INVALID_ARG, "problem.sched must be 4-byte aligned");
  if (p->total_tokens == 0) return FP_OK;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)p->head_dim);

  fp::AttnParams a;
  memset(&a, 0, sizeof a);
  const int64_t T = p->total_tokens;
  const int64_t kv_rows = c ? (int64_t)c->num_pages * c->page_size : T;  // rows of the K/V source
  if ((st = make_tmap(&a.tm_q, q, T, (int64_t)p->num_q_heads * p->head_dim, fp::kTileM, fp8)) != FP_OK) return st;
  if ((st = make_tmap(&a.tm_k, k, kv_rows, (int64_t)p->num_kv_heads * p->head_dim, p->block_size, fp8)) != FP_OK)
    return st;
  if ((st = make_tmap(&a.tm_v, v, kv_rows, (int64_t)p->num_kv_heads * p->head_dim, p->block_size)) != FP_OK) return st;
  a.seq = seq_info(p, c);
  a.hq = p->num_q_heads;
  a.hkv = p->num_kv_heads;
  a.group = p->num_q_heads / p->num_kv_heads;
  // exact tile count comes from the device tables; the grid uses an upper bound
  const long long tiles_ub = (long long)p->num_q_heads * ((T + fp::kTileM - 1) / fp::kTileM + p->num_seqs);
  a.num_tiles = 0;
  a.dense = dense;
  a.counts = counts;
  a.indices = indices;
  a.index_elems = index_elems(p, c);
  a.scale_log2 = scale * qk_scale * 1.4426950408889634f;
  a.fp8 = fp8 ? 1 : 0;
  a.q_exp = q_exp;
  a.k_exp = k_exp;
  a.sched = p->sched;
  a.out = static_cast<uint16_t*>(out);
  a.out32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 ? 1 : 0;
  a.lse = lse;
  a.dev_status = dev_status;
  a.wait_limit_ns = wait_limit_ns();
  // test hook (bounded-wait failure path): FP_TEST_UNSIGNALLED_WAIT=1 makes the softmax warps wait
  // on a barrier that nothing arrives on; the wait runs out, FP_DEV_TIMEOUT is set, the CTA unwinds
  const char* tw = getenv("FP_TEST_UNSIGNALLED_WAIT");
  a.test_unsignalled_wait = (tw && tw[0] == '1') ? 1 : 0;
  // tuning / test knob: FP_ATTN_UNITS=pairs or rows forces the attention schedule of the sparse call
  // (default: chosen on the device from the lists' density, for the plain bf16 prefill with B = 128).
  // The dense call always runs the paired schedule (the row kernel is not launched for it), so the
  // knob is not passed on there.
  const char* un = getenv("FP_ATTN_UNITS");
  a.units = dense ? 0 : (un && strcmp(un, "pairs") == 0) ? 1 : (un && strcmp(un, "rows") == 0) ? 2 : 0;
  const int grid = (int)(tiles_ub < sm_count() ? tiles_ub : sm_count());
  return cuda_status(fp::launch_attn(a, grid, static_cast<cudaStream_t>(stream)), "attention launch");
}

}  // namespace

namespace fp {
fp_status set_error(fp_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

unsigned long long context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrentFn>(a);
      get_id = reinterpret_cast<GetIdFn>(b);
    }
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

cudaError_t set_max_smem(const void* func, int bytes, unsigned long long (&done)[kMaxCachedDevices]) {
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool cached = dev >= 0 && dev < kMaxCachedDevices;
  std::lock_guard<std::mutex> lock(mu);
  if (cached) {
    const unsigned long long id = context_id();
    if (id != 0 && done[dev] == id) return cudaSuccess;
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cached) done[dev] = context_id();  // the call above made the context current
  return e;
}
}  // namespace fp

extern "C" {

fp_status fp_index_buffer_elems(const int32_t* host_seqlens, int32_t num_seqs, int32_t block_size,
                                int32_t num_q_heads, int64_t* out_elems) {
  if (!host_seqlens || !out_elems) return fail(FP_ERR_INVALID_ARG, "NULL argument to fp_index_buffer_elems");
  if (num_seqs < 1 || num_seqs > FP_MAX_SEQS)
    return fail(FP_ERR_INVALID_ARG, "num_seqs=%d outside [1, %d]", num_seqs, FP_MAX_SEQS);
  if (num_q_heads < 1) return fail(FP_ERR_INVALID_ARG, "num_q_heads=%d must be >= 1", num_q_heads);
  if (block_size != 64 && block_size != 128)
    return fail(FP_ERR_UNSUPPORTED, "block_size=%d (64 or 128)", block_size);
  int64_t idx = 0;
  for (int s = 0; s < num_seqs; ++s) {
    if (host_seqlens[s] < 0) return fail(FP_ERR_INVALID_ARG, "sequence %d has negative length %d", s, host_seqlens[s]);
    const int64_t nb = ((int64_t)host_seqlens[s] + block_size - 1) / block_size;
    idx += (int64_t)num_q_heads * nb * (nb + 1) / 2;
  }
  *out_elems = idx;
  return FP_OK;
}

fp_status fp_check_device_status(int32_t bits) {
  if (bits == 0) return FP_OK;
  const fp_status st = (bits & FP_DEV_TIMEOUT) ? FP_ERR_TIMEOUT : FP_ERR_INVALID_ARG;
  return fail(st, "device status 0x%x:%s%s%s%s", (unsigned)bits,
              (bits & FP_DEV_TIMEOUT) ? " a bounded wait gave up (outputs of that launch are undefined);" : "",
              (bits & FP_DEV_BAD_LIST) ? " an index-list entry or count was out of range (skipped);" : "",
              (bits & FP_DEV_BAD_PROBLEM) ? " device sequence tables disagreed with the problem (no work done);" : "",
              (bits & ~(FP_DEV_TIMEOUT | FP_DEV_BAD_LIST | FP_DEV_BAD_PROBLEM)) ? " unknown bits;" : "");
}

fp_status fp_problem_init(fp_problem* p, const int32_t* host_cu, int32_t num_seqs, const int32_t* dev_cu,
                          int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size) {
  if (!p || !host_cu || !dev_cu) return fail(FP_ERR_INVALID_ARG, "NULL argument to fp_problem_init");
  if (num_seqs < 1 || num_seqs > FP_MAX_SEQS)
    return fail(FP_ERR_INVALID_ARG, "num_seqs=%d outside [1, %d]", num_seqs, FP_MAX_SEQS);
  if (block_size != 64 && block_size != 128)
    return fail(FP_ERR_UNSUPPORTED, "block_size=%d (64 or 128)", block_size);
  if (host_cu[0] != 0) return fail(FP_ERR_INVALID_ARG, "cu_seqlens[0] must be 0");
  int64_t nb_tot = 0, idx = 0, max_nb = 0;
  for (int s = 0; s < num_seqs; ++s) {
    const int64_t L = (int64_t)host_cu[s + 1] - host_cu[s];
    if (L < 0) return fail(FP_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing (sequence %d)", s);
    const int64_t nb = (L + block_size - 1) / block_size;
    nb_tot += nb;
    idx += (int64_t)num_q_heads * nb * (nb + 1) / 2;
    if (nb > max_nb) max_nb = nb;
  }
  if (host_cu[num_seqs] > (int64_t)INT32_MAX / 2 || nb_tot > INT32_MAX)
    return fail(FP_ERR_INVALID_ARG, "too many tokens");
  memset(p, 0, sizeof *p);
  p->cu_seqlens = dev_cu;
  p->num_seqs = num_seqs;
  p->total_tokens = host_cu[num_seqs];
  p->total_blocks = (int32_t)nb_tot;
  p->max_seq_blocks = (int32_t)max_nb;
  p->index_elems = idx;
  p->num_q_heads = num_q_heads;
  p->num_kv_heads = num_kv_heads;
  p->head_dim = head_dim;
  p->block_size = block_size;
  return check_problem(p);
}

namespace {
fp_status pool_impl(const fp_problem* p, const fp_paged_cache* c, const void* q, const void* k, float* q_pool,
                    float* k_pool, void* stream) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if ((st = check_cache(p, c)) != FP_OK) return st;
  if (!q || !k || !q_pool || !k_pool) return fail(FP_ERR_INVALID_ARG, "q, k, q_pool and k_pool must be non-NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_pool) || !aligned16(k_pool))
    return fail(FP_ERR_INVALID_ARG, "q, k, q_pool and k_pool must be 16-byte aligned");
  if (p->total_blocks == 0) return FP_OK;
  fp::PoolParams a;
  a.seq = seq_info(p, c);
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.q_pool = q_pool;
  a.k_pool = k_pool;
  a.q_row = p->num_q_heads * p->head_dim;
  a.k_row = p->num_kv_heads * p->head_dim;
  a.q_chunks = (a.q_row + 1023) / 1024;
  a.k_chunks = (a.k_row + 1023) / 1024;
  a.dev_status = nullptr;
  const long long items = (long long)p->total_blocks * a.q_chunks + (long long)a.seq.total_kv_blocks * a.k_chunks;
  const long long cap = (long long)sm_count() * 16;
  const int grid = (int)(items < cap ? items : cap);
  return cuda_status(fp::launch_pool(a, grid, static_cast<cudaStream_t>(stream)), "pool launch");
}
}  // namespace

fp_status fp_block_pool(const fp_problem* p, const void* q, const void* k, float* q_pool, float* k_pool,
                        void* stream) {
  return pool_impl(p, nullptr, q, k, q_pool, k_pool, stream);
}

namespace {
fp::SearchParams search_params(const fp_problem* p, const fp_paged_cache* c, float tau, const float* k_pool,
                               int32_t* counts, int32_t* indices, int32_t* dev_status) {
  fp::SearchParams a;
  memset(&a, 0, sizeof a);
  a.seq = seq_info(p, c);
  a.k_pool = k_pool;
  a.hq = p->num_q_heads;
  a.hkv = p->num_kv_heads;
  a.group = p->num_q_heads / p->num_kv_heads;
  a.rows_blocks = 64 / a.group > 0 ? 64 / a.group : 1;
  // tiles = Hkv * sum_s ceil(nb_s / TI), counted on the device; the grid uses an upper bound
  a.num_tiles = (int32_t)((long long)p->num_kv_heads * (p->total_blocks / a.rows_blocks + p->num_seqs));
  a.inv_sqrt_d = 1.0f / std::sqrt((float)p->head_dim);
  a.keep_all = tau <= 0.f;
  a.log_tau = tau > 0.f ? (float)std::log((double)tau) : -INFINITY;
  a.counts = counts;
  a.indices = indices;
  a.index_elems = index_elems(p, c);
  a.dev_status = dev_status;
  a.wait_limit_ns = wait_limit_ns();
  return a;
}

fp_status search_impl(const fp_problem* p, const fp_paged_cache* c, const float* q_pool, const float* k_pool,
                      float tau, int32_t* counts, int32_t* indices, int32_t* dev_status, void* stream) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if ((st = check_cache(p, c)) != FP_OK) return st;
  if (!q_pool || !k_pool || !counts || !indices)
    return fail(FP_ERR_INVALID_ARG, "q_pool, k_pool, counts and indices must be non-NULL");
  if (!aligned16(q_pool) || !aligned16(k_pool)) return fail(FP_ERR_INVALID_ARG, "pooled tensors must be 16-byte aligned");
  if (!std::isfinite(tau)) return fail(FP_ERR_INVALID_ARG, "tau must be finite");
  const fp::KeySplitLayout kl = fp::key_split_layout(seq_info(p, c).total_kv_blocks, p->num_kv_heads);
  if (p->key_split) {
    if ((reinterpret_cast<uintptr_t>(p->key_split) & 255u) != 0)
      return fail(FP_ERR_INVALID_ARG, "problem.key_split must be 256-byte aligned");
    if (p->key_split_bytes < kl.total)
      return fail(FP_ERR_INVALID_ARG, "problem.key_split holds %lld bytes, this search needs %lld",
                  (long long)p->key_split_bytes, (long long)kl.total);
  }
  if (p->total_blocks == 0) return FP_OK;
  fp::SearchParams a = search_params(p, c, tau, k_pool, counts, indices, dev_status);
  a.q_pool = q_pool;
  if (p->key_split) {
    a.ksplit = static_cast<unsigned char*>(p->key_split);
    a.knorm2 = reinterpret_cast<float*>(static_cast<unsigned char*>(p->key_split) + kl.norms);
  }
  return cuda_status(fp::launch_search(a, static_cast<cudaStream_t>(stream)), "search launch");
}
}  // namespace

fp_status fp_key_split_bytes(const fp_problem* p, const fp_paged_cache* cache, int64_t* bytes) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if ((st = check_cache(p, cache)) != FP_OK) return st;
  if (!bytes) return fail(FP_ERR_INVALID_ARG, "bytes must be non-NULL");
  *bytes = fp::key_split_layout(seq_info(p, cache).total_kv_blocks, p->num_kv_heads).total;
  return FP_OK;
}

fp_status fp_block_search(const fp_problem* p, const float* q_pool, const float* k_pool, float tau,
                          int32_t* counts, int32_t* indices, int32_t* dev_status, void* stream) {
  return search_impl(p, nullptr, q_pool, k_pool, tau, counts, indices, dev_status, stream);
}

fp_status fp_block_search_topp(const fp_problem* p, const float* q_pool, const float* k_pool, float gamma,
                               float* scores, int32_t* counts, int32_t* indices, int32_t* dev_status,
                               void* stream) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if (!q_pool || !k_pool || !scores || !counts || !indices)
    return fail(FP_ERR_INVALID_ARG, "q_pool, k_pool, scores, counts and indices must be non-NULL");
  if (!aligned16(q_pool) || !aligned16(k_pool)) return fail(FP_ERR_INVALID_ARG, "pooled tensors must be 16-byte aligned");
  if (!std::isfinite(gamma)) return fail(FP_ERR_INVALID_ARG, "gamma must be finite");
  if (p->total_blocks == 0) return FP_OK;
  fp::SearchParams a = search_params(p, nullptr, gamma, k_pool, counts, indices, dev_status);
  a.q_pool = q_pool;
  return cuda_status(fp::launch_topp(a, gamma, scores, static_cast<cudaStream_t>(stream)), "top-p search launch");
}

fp_status fp_block_pool_search(const fp_problem* p, const void* q, const void* k, float tau, float* q_pool,
                               float* k_pool, int32_t* counts, int32_t* indices, int32_t* dev_status,
                               void* stream) {
  fp_status st = fp_block_pool(p, q, k, q_pool, k_pool, stream);
  if (st != FP_OK) return st;
  return fp_block_search(p, q_pool, k_pool, tau, counts, indices, dev_status, stream);
}

fp_status fp_block_sparse_attn(const fp_problem* p, const void* q, const void* k, const void* v,
                               const int32_t* counts, const int32_t* indices, float softmax_scale, void* out,
                               float* lse, int32_t* dev_status, void* stream) {
  return attn_common(p, nullptr, q, k, v, counts, indices, 0, softmax_scale, out, lse, dev_status, stream);
}

fp_status fp_dense_attn(const fp_problem* p, const void* q, const void* k, const void* v, float softmax_scale,
                        void* out, float* lse, int32_t* dev_status, void* stream) {
  return attn_common(p, nullptr, q, k, v, nullptr, nullptr, 1, softmax_scale, out, lse, dev_status, stream);
}

namespace {
fp_status check_fp8_scales(float q_scale, float k_scale, float* qk) {
  if (!std::isfinite(q_scale) || !std::isfinite(k_scale) || !(q_scale > 0.f) || !(k_scale > 0.f))
    return fail(FP_ERR_INVALID_ARG, "q_scale and k_scale must be finite and positive");
  *qk = q_scale * k_scale;
  if (!std::isfinite(*qk) || !(*qk > 0.f)) return fail(FP_ERR_INVALID_ARG, "q_scale * k_scale out of range");
  return FP_OK;
}
}  // namespace

fp_status fp_block_sparse_attn_fp8(const fp_problem* p, const void* q, const void* k, const void* v, float q_scale,
                                   float k_scale, const int32_t* counts, const int32_t* indices, float softmax_scale,
                                   void* out, float* lse, int32_t* dev_status, void* stream) {
  float qk = 1.f;
  fp_status st = check_fp8_scales(q_scale, k_scale, &qk);
  if (st != FP_OK) return st;
  return attn_common(p, nullptr, q, k, v, counts, indices, 0, softmax_scale, out, lse, dev_status, stream, true, qk);
}

fp_status fp_dense_attn_fp8(const fp_problem* p, const void* q, const void* k, const void* v, float q_scale,
                            float k_scale, float softmax_scale, void* out, float* lse, int32_t* dev_status,
                            void* stream) {
  float qk = 1.f;
  fp_status st = check_fp8_scales(q_scale, k_scale, &qk);
  if (st != FP_OK) return st;
  return attn_common(p, nullptr, q, k, v, nullptr, nullptr, 1, softmax_scale, out, lse, dev_status, stream, true,
                     qk);
}

fp_status fp_block_sparse_attn_fp8_blockscaled(const fp_problem* p, const void* q, const void* k, const void* v,
                                               const int8_t* q_exp, const int8_t* k_exp, const int32_t* counts,
                                               const int32_t* indices, float softmax_scale, void* out, float* lse,
                                               int32_t* dev_status, void* stream) {
  if (!q_exp || !k_exp) return fail(FP_ERR_INVALID_ARG, "q_exp and k_exp must be non-NULL");
  return attn_common(p, nullptr, q, k, v, counts, indices, 0, softmax_scale, out, lse, dev_status, stream, true, 1.f,
                     q_exp, k_exp);
}

fp_status fp_dense_attn_fp8_blockscaled(const fp_problem* p, const void* q, const void* k, const void* v,
                                        const int8_t* q_exp, const int8_t* k_exp, float softmax_scale, void* out,
                                        float* lse, int32_t* dev_status, void* stream) {
  if (!q_exp || !k_exp) return fail(FP_ERR_INVALID_ARG, "q_exp and k_exp must be non-NULL");
  return attn_common(p, nullptr, q, k, v, nullptr, nullptr, 1, softmax_scale, out, lse, dev_status, stream, true, 1.f,
                     q_exp, k_exp);
}

namespace {
struct WorkspaceLayout {
  int64_t q_pool, k_pool, counts, indices, sched, ksplit, total;  // byte offsets and total size
};
int64_t align256(int64_t x) { return (x + 255) & ~(int64_t)255; }
WorkspaceLayout workspace_layout(const fp_problem* p) {
  WorkspaceLayout w;
  const int64_t nb = p->total_blocks, d = p->head_dim;
  w.q_pool = 0;
  w.k_pool = align256(w.q_pool + nb * p->num_q_heads * d * 4);
  w.counts = align256(w.k_pool + nb * p->num_kv_heads * d * 4);
  w.indices = align256(w.counts + (int64_t)p->num_q_heads * nb * 4);
  w.sched = align256(w.indices + p->index_elems * 4);
  w.ksplit = align256(w.sched + FP_SCHED_WORDS * 4);
  w.total = w.ksplit + fp::key_split_layout(nb, p->num_kv_heads).total;
  return w;
}
}  // namespace

fp_status fp_sparse_prefill_workspace(const fp_problem* p, int64_t* bytes) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if (!bytes) return fail(FP_ERR_INVALID_ARG, "bytes must be non-NULL");
  *bytes = workspace_layout(p).total;
  return FP_OK;
}

fp_status fp_sparse_prefill(const fp_problem* p, const void* q, const void* k, const void* v, float tau,
                            float softmax_scale, void* workspace, int64_t workspace_bytes, void* out, float* lse,
                            int32_t* dev_status, void* stream) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  const WorkspaceLayout w = workspace_layout(p);
  if (!workspace) return fail(FP_ERR_INVALID_ARG, "workspace must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return fail(FP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < w.total)
    return fail(FP_ERR_INVALID_ARG, "workspace of %lld bytes is smaller than the %lld bytes needed",
                (long long)workspace_bytes, (long long)w.total);
  char* base = static_cast<char*>(workspace);
  float* q_pool = reinterpret_cast<float*>(base + w.q_pool);
  float* k_pool = reinterpret_cast<float*>(base + w.k_pool);
  int32_t* counts = reinterpret_cast<int32_t*>(base + w.counts);
  int32_t* indices = reinterpret_cast<int32_t*>(base + w.indices);
  // the work counter lives in the workspace (scratch between calls): zeroed here, in stream order
  fp_problem pw = *p;
  pw.sched = reinterpret_cast<int32_t*>(base + w.sched);
  pw.key_split = base + w.ksplit;
  pw.key_split_bytes = w.total - w.ksplit;
  if ((st = cuda_status(cudaMemsetAsync(pw.sched, 0, FP_SCHED_WORDS * sizeof(int32_t),
                                        static_cast<cudaStream_t>(stream)), "work counter reset")) != FP_OK)
    return st;
  if ((st = fp_block_pool(p, q, k, q_pool, k_pool, stream)) != FP_OK) return st;
  if ((st = fp_block_search(&pw, q_pool, k_pool, tau, counts, indices, dev_status, stream)) != FP_OK) return st;
  return fp_block_sparse_attn(&pw, q, k, v, counts, indices, softmax_scale, out, lse, dev_status, stream);
}

namespace {
fp_status validate_impl(const fp_problem* p, const fp_paged_cache* c, const int32_t* counts, const int32_t* indices,
                        int32_t* dev_status, void* stream) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if ((st = check_cache(p, c)) != FP_OK) return st;
  if (!counts || !indices || !dev_status)
    return fail(FP_ERR_INVALID_ARG, "counts, indices and dev_status must be non-NULL");
  if (p->total_blocks == 0) return FP_OK;
  fp::ValidateParams a;
  a.seq = seq_info(p, c);
  a.hq = p->num_q_heads;
  a.counts = counts;
  a.indices = indices;
  a.index_elems = index_elems(p, c);
  a.dev_status = dev_status;
  return cuda_status(fp::launch_validate(a, static_cast<cudaStream_t>(stream)), "validate launch");
}
}  // namespace

fp_status fp_validate_lists(const fp_problem* p, const int32_t* counts, const int32_t* indices, int32_t* dev_status,
                            void* stream) {
  return validate_impl(p, nullptr, counts, indices, dev_status, stream);
}

// ---- chunked prefill onto a paged key/value cache
fp_status fp_paged_cache_init(fp_paged_cache* c, const fp_problem* p, const int32_t* host_cu_seqlens,
                              const int32_t* host_prefix_lens, const int32_t* dev_prefix_lens,
                              const int32_t* dev_block_table, int32_t max_pages, int32_t page_size,
                              int32_t num_pages) {
  fp_status st = check_problem(p);
  if (st != FP_OK) return st;
  if (!c || !host_cu_seqlens || !host_prefix_lens || !dev_prefix_lens || !dev_block_table)
    return fail(FP_ERR_INVALID_ARG, "NULL argument to fp_paged_cache_init");
  const int B = p->block_size;
  if (page_size <= 0 || page_size % B)
    return fail(FP_ERR_UNSUPPORTED, "page_size=%d must be a positive multiple of block_size=%d", page_size, B);
  if (max_pages < 1 || num_pages < 1) return fail(FP_ERR_INVALID_ARG, "max_pages and num_pages must be >= 1");
  if ((int64_t)num_pages * page_size > (int64_t)INT32_MAX)
    return fail(FP_ERR_INVALID_ARG, "num_pages * page_size exceeds 2^31 - 1 rows");
  if (host_cu_seqlens[p->num_seqs] != p->total_tokens)
    return fail(FP_ERR_INVALID_ARG, "host_cu_seqlens does not match the problem");
  int64_t kb = 0, idx = 0;
  for (int s = 0; s < p->num_seqs; ++s) {
    const int64_t L = (int64_t)host_cu_seqlens[s + 1] - host_cu_seqlens[s];
    const int64_t P = host_prefix_lens[s];
    if (L < 0) return fail(FP_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing (sequence %d)", s);
    if (P < 0 || P % B)
      return fail(FP_ERR_INVALID_ARG, "prefix_lens[%d]=%lld must be a non-negative multiple of block_size=%d", s,
                  (long long)P, B);
    if ((P + L + page_size - 1) / page_size > max_pages)
      return fail(FP_ERR_INVALID_ARG, "sequence %d needs %lld pages, more than max_pages=%d", s,
                  (long long)((P + L + page_size - 1) / page_size), max_pages);
    const int64_t nb = (L + B - 1) / B, pb = P / B;
    kb += pb + nb;
    idx += (int64_t)p->num_q_heads * (nb * pb + nb * (nb + 1) / 2);
  }
  if (kb > INT32_MAX) return fail(FP_ERR_INVALID_ARG, "too many key blocks");
  memset(c, 0, sizeof *c);
  c->prefix_lens = dev_prefix_lens;
  c->block_table = dev_block_table;
  c->max_pages = max_pages;
  c->page_size = page_size;
  c->num_pages = num_pages;
  c->total_kv_blocks = (int32_t)kb;
  c->index_elems = idx;
  return FP_OK;
}

fp_status fp_paged_block_pool(const fp_problem* p, const fp_paged_cache* c, const void* q, const void* k_cache,
                              float* q_pool, float* k_pool, void* stream) {
  if (!c) return fail(FP_ERR_INVALID_ARG, "cache is NULL");
  return pool_impl(p, c, q, k_cache, q_pool, k_pool, stream);
}

fp_status fp_paged_block_search(const fp_problem* p, const fp_paged_cache* c, const float* q_pool,
                                const float* k_pool, float tau, int32_t* counts, int32_t* indices,
                                int32_t* dev_status, void* stream) {
  if (!c) return fail(FP_ERR_INVALID_ARG, "cache is NULL");
  return search_impl(p, c, q_pool, k_pool, tau, counts, indices, dev_status, stream);
}

fp_status fp_paged_block_sparse_attn(const fp_problem* p, const fp_paged_cache* c, const void* q,
                                     const void* k_cache, const void* v_cache, const int32_t* counts,
                                     const int32_t* indices, float softmax_scale, void* out, float* lse,
                                     int32_t* dev_status, void* stream) {
  if (!c) return fail(FP_ERR_INVALID_ARG, "cache is NULL");
  return attn_common(p, c, q, k_cache, v_cache, counts, indices, 0, softmax_scale, out, lse, dev_status, stream);
}

fp_status fp_paged_dense_attn(const fp_problem* p, const fp_paged_cache* c, const void* q, const void* k_cache,
                              const void* v_cache, float softmax_scale, void* out, float* lse, int32_t* dev_status,
                              void* stream) {
  if (!c) return fail(FP_ERR_INVALID_ARG, "cache is NULL");
  return attn_common(p, c, q, k_cache, v_cache, nullptr, nullptr, 1, softmax_scale, out, lse, dev_status, stream);
}

fp_status fp_paged_validate_lists(const fp_problem* p, const fp_paged_cache* c, const int32_t* counts,
                                  const int32_t* indices, int32_t* dev_status, void* stream) {
  if (!c) return fail(FP_ERR_INVALID_ARG, "cache is NULL");
  return validate_impl(p, c, counts, indices, dev_status, stream);
}

fp_status fp_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_mufu)))
    return fail(FP_ERR_INVALID_ARG, "x, y_poly and y_mufu must be non-NULL for n > 0");
  return cuda_status(fp::launch_exp2_selftest(x, y_poly, y_mufu, n, static_cast<cudaStream_t>(stream)),
                     "exp2 self-test launch");
}

const char* fp_last_error(void) { return g_err; }

int32_t fp_version(void) { return 500; }

}  // extern "C"
