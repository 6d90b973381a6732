// fp_seq.cuh -- per-launch sequence tables in shared memory (varlen packing).
//
// Every kernel starts by turning the device cu_seqlens (and, for a chunked prefill onto a cache,
// the prefix lengths) into prefix tables so that a global block id or tile id maps back to
// (sequence, local index) with a short binary search:
//   s_cu[s]   token offset of sequence s's queries       (s = 0..S)
//   s_cb[s]   first global query-block id of sequence s  (nb_s = ceil(L_s / B))
//   s_ct[s]   first tile id of sequence s                (tiles_s = mult * ceil(L_s / rows))
//   s_ib[s]   first index-list entry of sequence s       (sum_{s'<s} hq * (nb*pb + nb(nb+1)/2))
//   s_pb[s]   cached prefix blocks of sequence s         (prefix_s / B; 0 without a cache)
//   s_ckb[s]  first global key-block id of sequence s    (sum_{s'<s} pb + nb)
// Query block i of sequence s is key block s_pb[s] + i: its list row has room for pb + i + 1
// entries. The tables are checked against the host-side sizes; on mismatch the kernel flags
// kDevBadProblem and does no work, so a wrong cu_seqlens can never push a load out of bounds.
#pragma once
#include "fp_dev.cuh"
#include "fp_internal.h"

namespace fp {

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Must be called by every thread of the block. tile_rows <= 0 skips the tile table; s_ib may be
// null. Returns true when the tables are consistent with `si`.
static __device__ bool build_seq_tables(const SeqInfo& si, int* s_cu, int* s_cb, int* s_ct, long long* s_ib, int hq,
                                 int tile_rows, int tile_mult, int* s_ok, int32_t* dev_status, int* s_pb,
                                 int* s_ckb) {
  const int S = si.num_seqs;
  for (int t = threadIdx.x; t <= S; t += blockDim.x) {
    s_cu[t] = si.cu_seqlens[t];
    const int pre = (si.prefix_lens && t < S) ? si.prefix_lens[t] : 0;
    // a negative or unaligned prefix is marked -1 and fails the consistency check below
    s_pb[t] = (pre >= 0 && pre % si.block == 0) ? pre / si.block : -1;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (S + 31) / 32;
    const int a = lane * per, b = min(S, a + per);
    int ok = 1, nb_sum = 0, nt_sum = 0, kb_sum = 0;
    long long ib_sum = 0;
    for (int s = a; s < b; ++s) {
      const int L = s_cu[s + 1] - s_cu[s];
      if (L < 0 || s_pb[s] < 0) ok = 0;
      const int Lc = max(L, 0);
      const long long nb = (Lc + si.block - 1) / si.block, pb = max(s_pb[s], 0);
      nb_sum += (int)nb;
      kb_sum += (int)(pb + nb);
      ib_sum += (long long)hq * (nb * pb + nb * (nb + 1) / 2);
      if (tile_rows > 0) nt_sum += tile_mult * ((Lc + tile_rows - 1) / tile_rows);
    }
    const int nb_incl = warp_incl_scan(nb_sum);
    const int nt_incl = warp_incl_scan(nt_sum);
    const int kb_incl = warp_incl_scan(kb_sum);
    const long long ib_incl = warp_incl_scan(ib_sum);
    int nb_run = nb_incl - nb_sum, nt_run = nt_incl - nt_sum, kb_run = kb_incl - kb_sum;
    long long ib_run = ib_incl - ib_sum;
    for (int s = a; s < b; ++s) {
      s_cb[s] = nb_run;
      s_ckb[s] = kb_run;
      if (tile_rows > 0) s_ct[s] = nt_run;
      if (s_ib) s_ib[s] = ib_run;
      const int Lc = max(s_cu[s + 1] - s_cu[s], 0);
      const long long nb = (Lc + si.block - 1) / si.block, pb = max(s_pb[s], 0);
      nb_run += (int)nb;
      kb_run += (int)(pb + nb);
      ib_run += (long long)hq * (nb * pb + nb * (nb + 1) / 2);
      if (tile_rows > 0) nt_run += tile_mult * ((Lc + tile_rows - 1) / tile_rows);
    }
    ok = __all_sync(0xffffffffu, ok);
    const int nb_tot = __shfl_sync(0xffffffffu, nb_incl, 31);
    const int nt_tot = __shfl_sync(0xffffffffu, nt_incl, 31);
    const int kb_tot = __shfl_sync(0xffffffffu, kb_incl, 31);
    const long long ib_tot = __shfl_sync(0xffffffffu, ib_incl, 31);
    if (lane == 0) {
      s_cb[S] = nb_tot;
      s_ckb[S] = kb_tot;
      if (s_ib) s_ib[S] = ib_tot;
      if (tile_rows > 0) s_ct[S] = nt_tot;
      if (s_cu[0] != 0 || s_cu[S] != si.total_tokens || nb_tot != si.total_blocks || kb_tot != si.total_kv_blocks)
        ok = 0;
      *s_ok = ok;
      if (!ok && blockIdx.x == 0) dev_flag(dev_status, kDevBadProblem);
    }
  }
  __syncthreads();
  return *s_ok != 0;
}

// Largest s in [0, S) with tab[s] <= x (tab non-decreasing, tab[0] <= x < tab[S]).
__device__ __forceinline__ int find_seq(const int* tab, int S, int x) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Start of the index-list row (sequence s, q-head h, local query block i): row i holds up to
// pb + i + 1 entries (the key blocks 0 .. pb + i), pb = s_pb[s] (triangular layout when pb = 0).
__device__ __forceinline__ int64_t list_row(const int* s_cb, const long long* s_ib, const int* s_pb, int s, int h,
                                            int i) {
  const int64_t nb = s_cb[s + 1] - s_cb[s], pb = s_pb[s];
  return (int64_t)s_ib[s] + (int64_t)h * (nb * pb + nb * (nb + 1) / 2) + (int64_t)i * pb + (int64_t)i * (i + 1) / 2;
}

// Row of the key/value source holding key token u (0-based within sequence s's keys), or -1 when
// the block table points outside the cache (or u lies past the table's row): callers flag
// FP_DEV_BAD_PROBLEM and skip the load.
__device__ __forceinline__ long long kv_row(const SeqInfo& si, const int* s_cu, int s, int u) {
  if (!si.block_table) return (long long)s_cu[s] + u;
  const int lp = u / si.page_size;
  if (u < 0 || lp >= si.max_pages) return -1;
  const int page = __ldg(si.block_table + (long long)s * si.max_pages + lp);
  if (page < 0 || page >= si.num_pages) return -1;
  return (long long)page * si.page_size + u % si.page_size;
}

}  // namespace fp
