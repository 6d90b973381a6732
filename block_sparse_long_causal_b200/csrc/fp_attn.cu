// fp_attn.cu -- block-sparse (and dense) causal flash attention for sm_100a.
//
// FlashPrefill, skill summary page, "Architecture Overview" ("Physical Index Jumping": attention
// visits only the blocks named by the index lists) and the FlashPrefill V2 abstract (block-sparse
// prefill operator with warp specialisation; a dense baseline built the same way). The online
// softmax is the standard flash-attention recurrence.
//
// Design (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: Q tile (128 rows x 128 d, bf16, 128B swizzle, two 64-column slabs),
//               K and V tiles of B keys in rings of kStagesK / kStagesV slots; K/V coordinates
//               come straight from the index lists ("physical index jumping").
//   warp 1      tcgen05 issuer (one thread): S = Q K^T (M=128, N=B, K=16 steps) into TMEM, then
//               O += P V with P read from TMEM (A operand) and V from shared memory (MN-major B).
//               Owns the TMEM allocation (512 columns: S0 | S1 | O).
//   warps 2-5   softmax: thread r owns query row r of the tile (its TMEM lane). Loads S from TMEM,
//               applies the causal mask on diagonal tiles, keeps a running max in log2 units and
//               only rescales O (in TMEM) when the max grows by more than 2^8 (the stale max is
//               exact because numerator and denominator share it), writes P as bf16 into the S
//               columns it came from, and finally normalises O and stores it (and the LSE).
// S/P are double buffered so the QK^T of block n+1 overlaps the softmax of block n.
// GQA: tiles are ordered (query tile descending, then q-head), so the G q-heads sharing a kv-head
// run on neighbouring CTAs at the same time and their K/V tiles come from L2 after the first read.
// Block size 64: a 128-row tile holds two query blocks; the kv iteration is the ascending union of
// both lists, and a per-half bit masks rows of the block whose list lacks the current kv block.
// Every wait is bounded; on timeout the CTA flags FP_DEV_TIMEOUT, drains and returns.
#include "fp_internal.h"
#include "fp_seq.cuh"

namespace fp {

constexpr int kThreads = 192;
constexpr unsigned kFull = 0xffffffffu;
// Limit of the waits that only let already-issued copies / MMAs finish on the abort path.
constexpr uint64_t kDrainLimitNs = 1000000000ull;
// exp2 pairs (index mod 8) evaluated by the FMA-pipe polynomial instead of MUFU: 3 of 8
constexpr unsigned kPolyPairs = 0xA4u;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0, kTmemO = 256;

template <int BK>
struct Cfg {
  static constexpr int kStagesK = BK == 128 ? 3 : 4;
  static constexpr int kStagesV = BK == 128 ? 2 : 4;
  static constexpr uint32_t kQBytes = kTileM * kHeadDim * 2;        // 32 KB
  static constexpr uint32_t kKVBytes = BK * kHeadDim * 2;           // one K or V tile
  static constexpr uint32_t kSlabQ = kTileM * 128;                  // 64 cols x 2 B x rows
  static constexpr uint32_t kSlabKV = BK * 128;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffV = kOffK + kStagesK * kKVBytes;
  static constexpr uint32_t kOffBar = kOffV + kStagesV * kKVBytes;
  // barriers: q_full, q_empty, k_full[], k_empty[], v_full[], v_empty[], s_full[2], p_full[2],
  // o_done, o_final, drain, never (the test hook's barrier that nothing arrives on)
  static constexpr int kNumBars = 2 + 2 * kStagesK + 2 * kStagesV + 4 + 4;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;      // tmem base, abort flag, ok
  static constexpr uint32_t kOffTab = (kOffMisc + 16 + 15) & ~15u;
  static constexpr uint32_t kTabBytes = 3 * 4 * (kMaxSeqs + 1) + 8 * (kMaxSeqs + 1) + 16;
  static constexpr uint32_t kSmem = kOffTab + kTabBytes + 1024;     // + alignment slack
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, BK, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kHeadDim, 0, 1);
};

// ------------------------------------------------------------------------ tile schedule --------
struct Tile {
  int s, qt, h;     // sequence, 128-row query tile (local), q-head
  int row0;         // first token (global) of the tile
  int len;          // sequence length
  int nb;           // blocks of the sequence
  int gb0;          // global id of block 0 of the sequence
};

// Tile order inside a sequence: kv-head outermost, then query tile descending (longest causal rows
// first), then the G q-heads of that kv-head. The CTAs running at the same time then stream the
// K/V blocks of one kv-head, which stay in L2 while the G q-heads and neighbouring query tiles
// reuse them.
__device__ __forceinline__ Tile decode_tile(int t, const int* s_cu, const int* s_cb, const int* s_ct, int S,
                                            int hq, int group) {
  Tile x;
  x.s = find_seq(s_ct, S, t);
  const int local = t - s_ct[x.s];
  const int ntile = (s_ct[x.s + 1] - s_ct[x.s]) / hq;
  const int per_g = ntile * group;
  const int g = local / per_g, rem = local % per_g;
  x.qt = ntile - 1 - rem / group;
  x.h = g * group + rem % group;
  x.row0 = s_cu[x.s] + x.qt * kTileM;
  x.len = s_cu[x.s + 1] - s_cu[x.s];
  x.nb = s_cb[x.s + 1] - s_cb[x.s];
  x.gb0 = s_cb[x.s];
  return x;
}

// k-th tile of this CTA in a boustrophedon order over the grid (balances the descending sizes).
__device__ __forceinline__ int tile_of(int k) {
  const int g = gridDim.x;
  return k * g + ((k & 1) ? (g - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}

// ---------------------------------------------------------------------- kv iteration -----------
// Ascending union of up to two lists (A: query block a_blk, B: query block b_blk = a_blk + 1 when
// B == 64). Entries outside [0, own block] are skipped (and reported by the softmax role).
struct KvIter {
  const int32_t* la;
  const int32_t* lb;
  int na, nbn, ia, ib, lima, limb;
  bool dense;
  bool bad;

  __device__ __forceinline__ int peek(const int32_t* l, int n, int& i, int lim) {
    while (i < n) {
      const int x = dense ? i : __ldg(l + i);
      if (x >= 0 && x <= lim) return x;
      bad = true;
      ++i;
    }
    return 0x7fffffff;
  }
  __device__ __forceinline__ bool next(int& j, int& mask) {
    const int ja = peek(la, na, ia, lima);
    const int jb = peek(lb, nbn, ib, limb);
    if (ja == 0x7fffffff && jb == 0x7fffffff) return false;
    j = min(ja, jb);
    mask = (ja == j ? 1 : 0) | (jb == j ? 2 : 0);
    if (ja == j) ++ia;
    if (jb == j) ++ib;
    return true;
  }
};

template <int BK>
__device__ __forceinline__ KvIter make_iter(const AttnParams& p, const Tile& t, const int* s_cb, const long long* s_ib) {
  KvIter it;
  it.ia = it.ib = 0;
  it.bad = false;
  it.dense = p.dense != 0;
  constexpr int per = kTileM / BK;  // query blocks per tile
  const int a_blk = t.qt * per;
  const int b_blk = (per == 2 && a_blk + 1 < t.nb) ? a_blk + 1 : -1;
  it.lima = a_blk;
  it.limb = b_blk;
  if (it.dense) {
    it.la = it.lb = nullptr;
    it.na = a_blk + 1;
    it.nbn = b_blk >= 0 ? b_blk + 1 : 0;
  } else {
    const int NB = p.seq.total_blocks;
    it.la = p.indices + list_row(s_cb, s_ib, t.s, t.h, a_blk);
    it.na = min(max(__ldg(p.counts + (long long)t.h * NB + t.gb0 + a_blk), 0), a_blk + 1);
    if (b_blk >= 0) {
      it.lb = p.indices + list_row(s_cb, s_ib, t.s, t.h, b_blk);
      it.nbn = min(max(__ldg(p.counts + (long long)t.h * NB + t.gb0 + b_blk), 0), b_blk + 1);
    } else {
      it.lb = nullptr;
      it.nbn = 0;
    }
  }
  return it;
}

// ---------------------------------------------------------------------- the kernel -------------
template <int BK>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<BK>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  // barrier addresses
  const uint32_t b_q_full = bar0, b_q_empty = bar0 + 8;
  auto b_k_full = [&](int i) { return bar0 + 16 + 8 * i; };
  auto b_k_empty = [&](int i) { return bar0 + 16 + 8 * (C::kStagesK + i); };
  auto b_v_full = [&](int i) { return bar0 + 16 + 8 * (2 * C::kStagesK + i); };
  auto b_v_empty = [&](int i) { return bar0 + 16 + 8 * (2 * C::kStagesK + C::kStagesV + i); };
  const uint32_t b_s_full0 = bar0 + 16 + 8 * (2 * C::kStagesK + 2 * C::kStagesV);
  const uint32_t b_p_full0 = b_s_full0 + 16;
  const uint32_t b_o_done = b_p_full0 + 16, b_o_final = b_o_done + 8, b_drain = b_o_final + 8;
  const uint32_t b_never = b_drain + 8;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* s_ok = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
  int* s_cu = reinterpret_cast<int*>(smem + C::kOffTab);
  int* s_cb = s_cu + (kMaxSeqs + 1);
  int* s_ct = s_cb + (kMaxSeqs + 1);
  long long* s_ib = reinterpret_cast<long long*>(smem + C::kOffTab + 12 * (kMaxSeqs + 1) + 4);
  s_ib = reinterpret_cast<long long*>(((uintptr_t)s_ib + 7) & ~(uintptr_t)7);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.seq.num_seqs;

  if (threadIdx.x == 0) {
    mbar_init(b_q_full, 1);
    mbar_init(b_q_empty, 1);
    for (int i = 0; i < C::kStagesK; ++i) { mbar_init(b_k_full(i), 1); mbar_init(b_k_empty(i), 1); }
    for (int i = 0; i < C::kStagesV; ++i) { mbar_init(b_v_full(i), 1); mbar_init(b_v_empty(i), 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(b_s_full0 + 8 * i, 1); mbar_init(b_p_full0 + 8 * i, 128); }
    mbar_init(b_o_done, 1);
    mbar_init(b_o_final, 1);
    mbar_init(b_drain, 1);
    mbar_init(b_never, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), kTmemCols);
    tmem_relinquish();
  }
  const bool ok = build_seq_tables(p.seq, s_cu, s_cb, s_ct, s_ib, p.hq, kTileM, p.hq, s_ok, p.dev_status) &&
                  (p.dense || s_ib[S] == p.index_elems);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (!ok && threadIdx.x == 0 && !p.dense) dev_flag(p.dev_status, kDevBadProblem);
  const int num_tiles = ok ? s_ct[S] : 0;

  if (warp == 0) {
    // =========================================================== TMA producer
    if (lane == 0) {
      uint32_t kit = 0, vit = 0;  // loads issued into the K / V rings
      int tc = 0, tc_issued = 0;  // tiles started / Q loads issued
      bool qissued = false;
      bool fail = false;
      for (int k = 0;; ++k, ++tc) {
        const int t = tile_of(k);
        if (t >= num_tiles || fail) break;
        const Tile tl = decode_tile(t, s_cu, s_cb, s_ct, S, p.hq, p.group);
        const int g = tl.h / p.group;
        if (!mbar_wait(b_q_empty, (tc & 1) ^ 1, p.wait_limit_ns)) { fail = true; break; }
        mbar_arrive_expect_tx(b_q_full, C::kQBytes);
        tma_load_2d(sQ, &p.tm_q, b_q_full, tl.h * kHeadDim, tl.row0);
        tma_load_2d(sQ + C::kSlabQ, &p.tm_q, b_q_full, tl.h * kHeadDim + 64, tl.row0);
        ++tc_issued;
        qissued = true;
        KvIter itr = make_iter<BK>(p, tl, s_cb, s_ib);
        int j, mask, pending_v = -1;
        while (true) {
          const bool more = itr.next(j, mask);
          if (more) {  // K of this block
            const int st = kit % C::kStagesK;
            if (!mbar_wait(b_k_empty(st), ((kit / C::kStagesK) & 1) ^ 1, p.wait_limit_ns)) { fail = true; break; }
            mbar_arrive_expect_tx(b_k_full(st), C::kKVBytes);
            const uint32_t dst = sK + st * C::kKVBytes;
            const int y = tl.row0 - tl.qt * kTileM + j * BK;
            tma_load_2d(dst, &p.tm_k, b_k_full(st), g * kHeadDim, y);
            tma_load_2d(dst + C::kSlabKV, &p.tm_k, b_k_full(st), g * kHeadDim + 64, y);
            ++kit;
          }
          if (pending_v >= 0) {  // V of the previous block (consumed after the next QK^T)
            const int st = vit % C::kStagesV;
            if (!mbar_wait(b_v_empty(st), ((vit / C::kStagesV) & 1) ^ 1, p.wait_limit_ns)) { fail = true; break; }
            mbar_arrive_expect_tx(b_v_full(st), C::kKVBytes);
            const uint32_t dst = sV + st * C::kKVBytes;
            const int y = tl.row0 - tl.qt * kTileM + pending_v * BK;
            tma_load_2d(dst, &p.tm_v, b_v_full(st), g * kHeadDim, y);
            tma_load_2d(dst + C::kSlabKV, &p.tm_v, b_v_full(st), g * kHeadDim + 64, y);
            ++vit;
          }
          if (!more) break;
          pending_v = j;
          if (*s_abort) { fail = true; break; }
        }
      }
      if (fail) {
        *s_abort = 1;
        dev_flag(p.dev_status, kDevTimeout);
        // let issued copies land before the CTA can exit (own, generous limit: copies always land)
        for (int i = 0; i < C::kStagesK; ++i) {
          const uint32_t n = kit > (uint32_t)i ? (kit - 1 - i) / C::kStagesK : 0;
          if (kit > (uint32_t)i) mbar_wait(b_k_full(i), n & 1, kDrainLimitNs);
        }
        for (int i = 0; i < C::kStagesV; ++i) {
          const uint32_t n = vit > (uint32_t)i ? (vit - 1 - i) / C::kStagesV : 0;
          if (vit > (uint32_t)i) mbar_wait(b_v_full(i), n & 1, kDrainLimitNs);
        }
        if (qissued) mbar_wait(b_q_full, (uint32_t)(tc_issued - 1) & 1, kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // =========================================================== tcgen05 issuer
    if (lane == 0) {
      uint32_t it = 0, vit = 0;
      int tc = 0;
      bool fail = false;
      auto pv = [&](uint32_t m, bool first) -> bool {
        const uint32_t b = m & 1;
        if (!mbar_wait(b_p_full0 + 8 * b, (m >> 1) & 1, p.wait_limit_ns)) return false;
        const int st = vit % C::kStagesV;
        if (!mbar_wait(b_v_full(st), (vit / C::kStagesV) & 1, p.wait_limit_ns)) return false;
        tc_fence_after();
        const uint32_t vbase = sV + st * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(vbase + kk * 2048, C::kSlabKV, 1024);
          mma_ts(tmem + kTmemO, tmem + kTmemS + 128 * b + kk * 8, bdesc, C::kIdescPV, (!first || kk > 0) ? 1u : 0u);
        }
        mma_commit(b_v_empty(st));
        mma_commit(b_o_done);
        ++vit;
        return true;
      };
      for (int k = 0;; ++k, ++tc) {
        const int t = tile_of(k);
        if (t >= num_tiles || fail) break;
        const Tile tl = decode_tile(t, s_cu, s_cb, s_ct, S, p.hq, p.group);
        KvIter itr = make_iter<BK>(p, tl, s_cb, s_ib);
        if (!mbar_wait(b_q_full, tc & 1, p.wait_limit_ns)) { fail = true; break; }
        tc_fence_after();
        int j, mask, n = 0;
        bool more = itr.next(j, mask);
        while (more) {
          const int st = it % C::kStagesK;
          if (!mbar_wait(b_k_full(st), (it / C::kStagesK) & 1, p.wait_limit_ns)) { fail = true; break; }
          tc_fence_after();
          const uint32_t b = it & 1;
          const uint32_t kbase = sK + st * C::kKVBytes;
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk) {
            const uint32_t koff = (kk & 3) * 32;  // 16 bf16 = 32 bytes inside the swizzle atom
            const uint64_t adesc = sdesc_sw128(sQ + (kk >> 2) * C::kSlabQ + koff, 16, 1024);
            const uint64_t bdesc = sdesc_sw128(kbase + (kk >> 2) * C::kSlabKV + koff, 16, 1024);
            mma_ss(tmem + kTmemS + 128 * b, adesc, bdesc, C::kIdescQK, kk > 0 ? 1u : 0u);
          }
          mma_commit(b_s_full0 + 8 * b);
          mma_commit(b_k_empty(st));
          more = itr.next(j, mask);
          if (!more) mma_commit(b_q_empty);
          if (n > 0 && !pv(it - 1, n == 1)) { fail = true; break; }
          ++it;
          ++n;
          if (*s_abort) { fail = true; break; }
        }
        if (fail) break;
        if (n > 0) {
          if (!pv(it - 1, n == 1)) { fail = true; break; }
          mma_commit(b_o_final);
        } else {
          mma_commit(b_q_empty);  // empty list: release Q without touching O
        }
      }
      if (fail) {
        *s_abort = 1;
        dev_flag(p.dev_status, kDevTimeout);
      }
      // all issued MMAs complete before TMEM is released (own, generous limit: MMAs always finish)
      mma_commit(b_drain);
      mbar_wait(b_drain, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else {
    // =========================================================== softmax / correction / epilogue
    const int q4 = warp & 3;                  // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;             // row of the tile owned by this thread
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int half = r / BK;                  // query block (within the tile) of this row
    uint32_t it = 0;
    int fc = 0;  // tiles with a non-empty kv list (phases of o_final)
    bool fail = false;
    bool bad_list = false;
    if (p.test_unsignalled_wait && num_tiles > 0)
      fail = __any_sync(kFull, !mbar_wait(b_never, 0, p.wait_limit_ns));
    for (int k = 0;; ++k) {
      const int t = tile_of(k);
      if (t >= num_tiles || fail) break;
      const Tile tl = decode_tile(t, s_cu, s_cb, s_ct, S, p.hq, p.group);
      KvIter itr = make_iter<BK>(p, tl, s_cb, s_ib);
      const int qpos = tl.qt * kTileM + r;    // local query position of this row
      float m_run = -INFINITY, l_run = 0.f;
      int j, mask, n = 0;
      while (itr.next(j, mask)) {
        const uint32_t b = it & 1;
        // tcgen05.ld/st are warp-collective: every branch around them is made warp-uniform
        if (__any_sync(kFull, !mbar_wait(b_s_full0 + 8 * b, (it >> 1) & 1, p.wait_limit_ns))) { fail = true; break; }
        tc_fence_after();
        uint32_t sr[BK];
#pragma unroll
        for (int c = 0; c < BK; c += 32)
          tmem_ld32(tmem + lane_off + kTmemS + 128 * b + c, *reinterpret_cast<uint32_t(*)[32]>(&sr[c]));
        tmem_wait_ld();
        // causal mask (diagonal tiles) and the per-half list mask (B = 64)
        const int valid = ((mask >> (kTileM / BK == 2 ? half : 0)) & 1) ? (qpos - j * BK) : -1;
        const bool masked = valid < BK - 1;   // this row needs element masking on this tile
        float mx;
        if (masked) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < BK; ++c) {
            const float v = (c <= valid) ? __uint_as_float(sr[c]) : -INFINITY;
            sr[c] = __float_as_uint(v);
            m4[c & 3] = fmaxf(m4[c & 3], v);
          }
          mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        } else {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < BK; c += 8) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
              m4[a] = fmax3(m4[a], __uint_as_float(sr[c + 2 * a]), __uint_as_float(sr[c + 2 * a + 1]));
          }
          mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        }
        const float m_tile = mx * p.scale_log2;
        const float m_new = fmaxf(m_run, m_tile);
        // grow the reference max only when it rises by more than 2^8 (lazy rescale); the stale
        // max is exact because the numerator and the denominator share it
        const bool grow = m_new > m_run + 8.0f;
        float alpha = 1.f;
        if (grow) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        l_run *= alpha;
        if (n > 0 && __any_sync(kFull, grow)) {
          // O must hold PV_{n-1} before it is rescaled (lanes that did not grow scale by 1)
          if (__any_sync(kFull, !mbar_wait(b_o_done, (it - 1) & 1, p.wait_limit_ns))) { fail = true; break; }
          tc_fence_after();
          const uint64_t a2 = f2_make(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < kHeadDim; c += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + kTmemO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float lo, hi;
              f2_split(fmul2(f2_bits(o[e], o[e + 1]), a2), lo, hi);
              o[e] = __float_as_uint(lo);
              o[e + 1] = __float_as_uint(hi);
            }
            tmem_st32(tmem + lane_off + kTmemO + c, o);
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        const uint64_t scale2 = f2_make(p.scale_log2, p.scale_log2);
        const uint64_t negm2 = f2_make(-m_use, -m_use);
        uint64_t sum2[2] = {0ull, 0ull};
        uint32_t pk[BK / 2];
        if (masked) {
          // exact zeros for masked keys: MUFU ex2(-inf) = 0
#pragma unroll
          for (int c = 0; c < BK; c += 2) {
            float x0, x1;
            f2_split(ffma2(f2_bits(sr[c], sr[c + 1]), scale2, negm2), x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            sum2[(c >> 1) & 1] = fadd2(sum2[(c >> 1) & 1], f2_make(p0, p1));
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
        } else {
          // split exp2 between MUFU and the FMA-pipe polynomial (pairs whose index has a bit in
          // kPolyPairs use the polynomial) so that neither unit alone bounds the softmax
#pragma unroll
          for (int c = 0; c < BK; c += 2) {
            const uint64_t x2 = ffma2(f2_bits(sr[c], sr[c + 1]), scale2, negm2);
            uint64_t p2;
            if ((kPolyPairs >> ((c >> 1) & 7)) & 1) {
              p2 = exp2_poly2(x2);
            } else {
              float x0, x1;
              f2_split(x2, x0, x1);
              p2 = f2_make(ex2_approx(x0), ex2_approx(x1));
            }
            sum2[(c >> 1) & 1] = fadd2(sum2[(c >> 1) & 1], p2);
            float p0, p1;
            f2_split(p2, p0, p1);
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
        }
        {
          float a0, a1, b0, b1;
          f2_split(sum2[0], a0, a1);
          f2_split(sum2[1], b0, b1);
          l_run += (a0 + a1) + (b0 + b1);
        }
#pragma unroll
        for (int c = 0; c < BK / 2; c += 32)
          tmem_st32(tmem + lane_off + kTmemS + 128 * b + c, *reinterpret_cast<uint32_t(*)[32]>(&pk[c]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p_full0 + 8 * b);
        ++it;
        ++n;
      }
      bad_list |= itr.bad;
      if (__any_sync(kFull, fail || *s_abort)) { fail = true; break; }
      const bool row_ok = qpos < tl.len;
      if (n == 0) {  // empty kv list (malformed input): zero output, LSE -inf
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((long long)(tl.row0 + r) * p.hq + tl.h) * kHeadDim);
          for (int c = 0; c < kHeadDim / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[(long long)tl.h * p.seq.total_tokens + tl.row0 + r] = -INFINITY;
        }
        continue;
      }
      // ---- epilogue: O / l -> bf16, LSE
      if (__any_sync(kFull, !mbar_wait(b_o_final, fc & 1, p.wait_limit_ns))) { fail = true; break; }
      ++fc;
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      uint16_t* orow = p.out + ((long long)(tl.row0 + r) * p.hq + tl.h) * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < kHeadDim; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + kTmemO + c, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
          dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
        }
      }
      if (row_ok && p.lse) {
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        p.lse[(long long)tl.h * p.seq.total_tokens + tl.row0 + r] =
            l_run > 0.f ? (m_use + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      }
      tc_fence_before();
    }
    if (fail) {
      *s_abort = 1;
      dev_flag(p.dev_status, kDevTimeout);
    }
    if (bad_list && r == 0) dev_flag(p.dev_status, kDevBadList);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int BK>
static cudaError_t launch_attn_t(const AttnParams& p, int grid, cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel<BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<BK>::kSmem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  attn_kernel<BK><<<grid, kThreads, Cfg<BK>::kSmem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_attn(const AttnParams& p, int grid, cudaStream_t st) {
  if (p.seq.block == 128) return launch_attn_t<128>(p, grid, st);
  return launch_attn_t<64>(p, grid, st);
}

}  // namespace fp
