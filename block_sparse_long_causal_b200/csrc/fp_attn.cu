// fp_attn.cu -- block-sparse (and dense) causal flash attention for sm_100a.
//
// FlashPrefill, skill summary page, "Architecture Overview" ("Physical Index Jumping": attention
// visits only the blocks named by the index lists) and the FlashPrefill V2 abstract (block-sparse
// prefill operator with PackGQA memory access, warp specialisation and pingpong pipelining; a dense
// baseline built the same way). The online softmax is the standard flash-attention recurrence.
//
// Design (one persistent CTA per SM, 12 warps in three warpgroups):
//   WG0  warp 0: TMA producer. Per work unit two Q tiles (128 rows x 128 d, bf16, 128B swizzle),
//                then K and V tiles of B keys in rings of kStages slots; K/V coordinates come
//                straight from the index lists ("physical index jumping").
//        warp 1: allocates 512 TMEM columns (S0 | S1 | O0 | O1) and issues tcgen05.mma from one
//                thread: S_k = Q_k K^T (M=128, N=B, K=16 steps, both operands K-major SW128 smem
//                descriptors) and O_k += P_k V (P_k read from TMEM as the A operand, V an MN-major
//                SW128 descriptor), in the pingpong order PV0(n-1) QK0(n) PV1(n-1) QK1(n).
//        warps 2-3: idle (they only give their registers to the softmax warpgroups).
//   WG1, WG2  softmax of slot 0 / slot 1: thread r owns query row r of its slot's tile (its TMEM
//                lane): tcgen05.ld of S, causal mask on diagonal tiles, running max in log2 units
//                (no max pass on unmasked items once the row has one), exp2 on MUFU (an FMA-pipe
//                polynomial share measured slower: it lengthens the softmax's dependency chains more
//                than it relieves MUFU), P packed to bf16 back into the S columns, lazy O rescale
//                (only when the max grows by more than 2^8), final normalisation and the bf16 store
//                of O and the LSE.
// Registers: setmaxnreg moves WG0 down to 104 and WG1/WG2 up to 200 per thread
// (128*104 + 256*200 = 384*168, the launch allocation of __launch_bounds__(384, 1)).
//
// A work unit pairs two Q tiles that read the same K/V stream, so a K/V tile both need is loaded
// once into shared memory for both (GQA packing): query tiles (2m+1, 2m) of one q-head (the last
// tile of an odd count runs alone). Each slot walks its own lists (two per slot when B = 64, where a
// 128-row tile holds two query blocks); a block both slots hold is one item for both, a block of one
// slot an item of that slot alone (the other skips its QK, PV and softmax), and a per-(slot, half)
// bit masks rows whose list lacks the item's block, so different lists stay exact. Single-slot
// items alternate between the slots wherever that loses no shared block, and a slot's QK is issued
// ahead of the other slot's pending PV, so one slot's softmax overlaps the other's MMAs whether the
// items are shared or not.
// Because QK_k(n) is issued after PV_k(n-1) and tcgen05.commit tracks all earlier MMAs, a slot
// that sees S_k(n) may rescale O_k without waiting: PV_k(n-1) has already completed.
// Units are ordered kv-head outermost, then by descending query tile, so concurrent CTAs stream
// the K/V of one kv-head (L2 resident) and the longest causal rows start first. With a work counter
// (fp_problem.sched) each CTA takes the next untaken unit of that order when its producer is free,
// which keeps the grid balanced for lists of any lengths (a load model of the 128K workload puts
// the busiest SM of a fixed share 4-15% above the mean, more the sparser the lists).
// A second schedule, for sparse lists (plain bf16 prefill, B = 128; see "row schedule" below), runs
// one query tile per unit with both softmax warpgroups on the same tile, each on half of every
// item's keys, and alternates two S buffers between items; the kernel picks it when fewer than 40% of
// the causal blocks are kept.
// Every wait is bounded; on timeout the CTA flags FP_DEV_TIMEOUT, lets issued copies and MMAs
// finish, frees TMEM and returns.
// Instances (template flags): kCache -- chunked prefill onto a (paged) K/V cache: each K/V block's
// TMA row comes from the block table and a query's causal limit is its key position (cached prefix
// + local position); the plain prefill is compiled without it. kFp8 -- e4m3 Q and K: their tiles
// are single 128-byte-row slabs loaded as uint8 boxes and Q K^T runs as kind::f8f6f4 (K = 32 per
// MMA); V, P and O stay bf16. Per-tensor scales are folded into the softmax scale; per-block
// power-of-two scales multiply it per row (query block) and per item (key block).
#include "fp_internal.h"
#include "fp_seq.cuh"

namespace fp {

constexpr int kThreads = 384;
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kTmemCols = 512;
constexpr int kRegsCtl = 104;       // WG0 (producer, MMA, idle)
constexpr int kRegsSoftmax = 200;  // WG1, WG2
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax == kThreads * 168,
              "register split must equal the launch allocation");
// Limit of the waits that only let already-issued copies / MMAs finish on the abort path.
constexpr uint64_t kDrainLimitNs = 1000000000ull;
// Item ring: the producer merges the index lists once and publishes, per unit, the unit's index,
// then each kv item as (block << 4 | row-mask bits), then kItemEnd; after its last unit, kUnitsEnd.
// Each entry has a full and an empty mbarrier: the MMA thread and every softmax warp arrive on the
// empty barrier once they have read the entry, and the producer waits on it before writing the
// entry's next use, so no reader can be overrun however far it lags.
constexpr int kRing = 32;
constexpr int kRingReaders = 9;  // the MMA thread and the 8 softmax warps
constexpr int kItemEnd = -1;
constexpr int kUnitsEnd = -2;
// Largest row sum of one item that the fast path (no max pass) accepts; see the softmax loop.
constexpr float kFastSumLimit = 65536.f;

// 2^e as a float for e in [-126, 127] (the per-block FP8 exponents lie in [-64, 64]): exact, so the
// scaled logit equals ldexpf's
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }
__device__ __forceinline__ uint32_t tmem_s(int k) { return 128u * k; }
__device__ __forceinline__ uint32_t tmem_o(int k) { return 256u + 128u * k; }

// kFp8: Q and K are e4m3 (1 byte per element: a 128-element head row is one 128-byte swizzle
// atom wide, so their tiles are a single slab); V and P stay bf16.
template <int BK, bool kFp8 = false>
struct Cfg {
  static constexpr int kStages = BK == 128 ? 2 : 4;                // K ring and V ring slots
  static constexpr uint32_t kQKEl = kFp8 ? 1 : 2;                   // bytes per Q / K element
  static constexpr uint32_t kQBytes = kTileM * kHeadDim * kQKEl;    // one Q slot
  static constexpr uint32_t kKBytes = BK * kHeadDim * kQKEl;        // one K tile
  static constexpr uint32_t kVBytes = BK * kHeadDim * 2;            // one V tile
  static constexpr uint32_t kSlabQ = kTileM * 128;                  // 128-byte rows x rows
  static constexpr uint32_t kSlabK = BK * 128;
  static constexpr uint32_t kSlabKV = BK * 128;                     // V slab (64 bf16 columns)
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = 2 * kQBytes;
  static constexpr uint32_t kOffV = kOffK + kStages * kKBytes;
  static constexpr uint32_t kOffBar = kOffV + kStages * kVBytes;
  // barriers: q_full, q_empty, k_full[], k_empty[], v_full[], v_empty[], s_full[2], p_full[2],
  // o_final[2], drain, never (the test hook's barrier that nothing arrives on), item_full[kRing],
  // item_empty[kRing]
  static constexpr int kNumBars = 2 + 4 * kStages + 6 + 2 + 2 * kRing;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;      // tmem base, abort flag, ok
  static constexpr uint32_t kOffRing = kOffMisc + 16;               // kRing int32 item entries
  static constexpr uint32_t kOffTab = (kOffRing + 4 * kRing + 15) & ~15u;
  // sequence tables (5 int arrays and one int64 array of num_seqs + 1 entries), sized per launch so
  // that the shared memory left to L1 does not shrink for the common few-sequence case
  static constexpr uint32_t tab_bytes(int num_seqs) { return 5 * 4 * (num_seqs + 1) + 8 * (num_seqs + 1) + 16; }
  static constexpr uint32_t smem_bytes(int num_seqs) { return kOffTab + tab_bytes(num_seqs) + 1024; }  // + alignment
  static constexpr uint32_t kSmemMax = smem_bytes(kMaxSeqs);
  static_assert(kSmemMax <= 227 * 1024, "shared memory per CTA");
  static constexpr uint32_t kIdescQK = kFp8 ? idesc_e4m3_f32(128, BK) : idesc_bf16_f32(128, BK, 0, 0);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kHeadDim, 0, 1);
};

// ------------------------------------------------------------------------ work units ----------
struct Unit {
  int s, g;         // sequence, kv-head
  int nslot;        // 1 or 2 active Q slots
  int qt[2], h[2];  // per slot: 128-row query tile (local), q-head
  int seq0;         // first query token of the sequence
  int len, nb, gb0; // query tokens of the sequence, its query blocks, global id of its block 0
  int pb;           // cached prefix blocks: query block i is key block pb + i
};

// Unit order inside a sequence: kv-head outermost, then descending query-tile pair, then the
// q-heads of that kv-head. A unit holds query tiles (2m+1, 2m) of one q-head (the last tile of an odd
// count runs alone): neighbouring query tiles of a head keep nearly the same key blocks (the sink,
// the vertical and slash structure repeat from tile to tile), so at sparse settings their lists
// overlap more than those of two heads at one tile do, and at density 1 they share every block but
// the upper tile's diagonal.
__device__ __forceinline__ Unit decode_unit(int t, const int* s_cu, const int* s_cb, const int* s_ct,
                                            const int* s_pb, int S, int group) {
  Unit u;
  u.s = find_seq(s_ct, S, t);
  const int local = t - s_ct[u.s];
  u.seq0 = s_cu[u.s];
  u.len = s_cu[u.s + 1] - u.seq0;
  u.nb = s_cb[u.s + 1] - s_cb[u.s];
  u.gb0 = s_cb[u.s];
  u.pb = s_pb[u.s];
  const int ntile = (u.len + kTileM - 1) / kTileM;
  const int np = (ntile + 1) / 2;
  const int per_g = np * group;
  u.g = local / per_g;
  const int rem = local % per_g;
  const int m = np - 1 - rem / group;
  const int h = u.g * group + rem % group;
  u.h[0] = u.h[1] = h;
  if (2 * m + 1 < ntile) {
    u.nslot = 2;
    u.qt[0] = 2 * m + 1;
    u.qt[1] = 2 * m;
  } else {
    u.nslot = 1;
    u.qt[0] = u.qt[1] = 2 * m;
  }
  return u;
}

// Unit schedule. Every CTA starts with unit blockIdx.x. With a work counter (p.sched) each further
// unit is the next one in the global order that no CTA has taken yet (greedy: a CTA that finishes
// early takes more, so the grid ends together whatever the lists' lengths); without one, the k-th
// unit of the CTA follows a boustrophedon order over the grid (balanced only for causal-dense sizes).
// The global order keeps the CTAs on neighbouring units either way: one kv-head's K/V at a time.
__device__ __forceinline__ int unit_of(int k) {
  const int g = gridDim.x;
  return k * g + ((k & 1) ? (g - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}
__device__ __forceinline__ int next_unit(int* sched, int k) {
  return sched ? (int)gridDim.x + atomicAdd(sched, 1) : unit_of(k);
}
// Called once per CTA after its last fetch: the grid's last CTA returns both counter words to zero
// (no fetch of this launch can follow), so launches ordered on a stream share the counter.
__device__ __forceinline__ void sched_release(int* sched) {
  if (!sched) return;
  __threadfence();
  if (atomicAdd(sched + 1, 1) == (int)gridDim.x - 1) {
    __threadfence();
    atomicExch(sched, 0);
    atomicExch(sched + 1, 0);
  }
}

// ---------------------------------------------------------------------- kv iteration -----------
// One index list of a slot (a 128-row tile holds two query blocks, so two lists, when B = 64).
// Scalar fields only, so that the walk stays in the producer thread's registers.
struct ListIter {
  const int32_t* l;
  int n, i, lim;
  int cur;  // valid entry at i (0x7fffffff past the end)
  int nxt;  // raw entry at i + 1, loaded one step ahead (0x7fffffff past the end)
  bool dense;

  __device__ __forceinline__ int raw(int k) const { return k < n ? (dense ? k : __ldg(l + k)) : 0x7fffffff; }
  // step to the next valid entry (entries outside [0, lim] are skipped and reported through bad);
  // the entry after it is loaded now and used at the next step, so the walk waits on no load
  __device__ __forceinline__ void advance(bool& bad) {
    ++i;
    int x = nxt;
    while (i < n && !(x >= 0 && x <= lim)) {
      bad = true;
      ++i;
      x = raw(i);
    }
    cur = i < n ? x : 0x7fffffff;
    nxt = raw(i + 1);
  }
  __device__ __forceinline__ void start(const int32_t* list, int count, int last, bool is_dense, bool& bad) {
    l = list;
    n = count;
    lim = last;
    dense = is_dense;
    i = -1;
    nxt = raw(0);
    advance(bad);
  }
};

// A slot's blocks: the ascending union of its lists.
struct SlotIter {
  ListIter a, b;

  __device__ __forceinline__ int first() const { return min(a.cur, b.cur); }
  // the slot's block after first() (nxt is unchecked: it only steers the order of the two slots)
  __device__ __forceinline__ int second() const {
    if (a.cur == b.cur) return min(a.nxt, b.nxt);
    return a.cur < b.cur ? min(a.nxt, b.cur) : min(b.nxt, a.cur);
  }
  // take block j (== first()): the bits of the lists that hold it
  __device__ __forceinline__ int pop(int j, bool& bad) {
    int hm = 0;
    if (a.cur == j) {
      hm = 1;
      a.advance(bad);
    }
    if (b.cur == j) {
      hm |= 2;
      b.advance(bad);
    }
    return hm;
  }
};

// The unit's item order. A block that both slots' lists hold is one item for both (its K/V tiles
// are loaded once). A block of one slot only is an item of that slot alone; the MMA issuer then
// overlaps that slot's softmax with the other slot's MMAs only if the next items alternate between
// the slots, so when the ascending union would give the same slot two single items in a row, the
// other slot's next block goes first whenever it is certainly not in the first slot's list (it lies
// strictly between that list's next two entries), which keeps every shared block shared.
struct KvIter {
  SlotIter s0, s1;
  int last;  // slot (0/1) of the previous single-slot item, -1 after a shared item or at the start
  bool bad;

  __device__ __forceinline__ bool next(int& j, int& mask) {
    const int a = s0.first(), b = s1.first();
    if (a == 0x7fffffff && b == 0x7fffffff) return false;
    if (a == b) {
      j = a;
      mask = s0.pop(a, bad) | (s1.pop(a, bad) << 2);
      last = -1;
      return true;
    }
    int pick = a < b ? 0 : 1;
    if (pick == last && a != 0x7fffffff && b != 0x7fffffff) {
      if (pick == 0 ? (b < s0.second()) : (a < s1.second())) pick ^= 1;
    }
    if (pick == 0) {
      j = a;
      mask = s0.pop(a, bad);
    } else {
      j = b;
      mask = s1.pop(b, bad) << 2;
    }
    last = pick;
    return true;
  }
};

template <int BK, bool kCache>
__device__ __forceinline__ void start_list(ListIter& it, const AttnParams& p, const Unit& u, int k, int hf,
                                           const int* s_cb, const long long* s_ib, const int* s_pb, bool& bad) {
  constexpr int per = kTileM / BK;  // query blocks per tile
  const int blk = u.qt[k] * per + hf;
  const bool exists = k < u.nslot && hf < per && blk < u.nb;
  const int jd = (kCache ? u.pb : 0) + blk;  // the query block's diagonal key block
  const int32_t* list = nullptr;
  int n = 0;
  if (exists) {
    if (p.dense) {
      n = jd + 1;
    } else {
      list = p.indices + list_row(s_cb, s_ib, s_pb, u.s, u.h[k], blk);
      n = min(max(__ldg(p.counts + (long long)u.h[k] * p.seq.total_blocks + u.gb0 + blk), 0), jd + 1);
    }
  }
  it.start(list, n, jd, p.dense != 0, bad);
}

template <int BK, bool kCache>
__device__ __forceinline__ KvIter make_iter(const AttnParams& p, const Unit& u, const int* s_cb,
                                            const long long* s_ib, const int* s_pb) {
  KvIter it;
  it.last = -1;
  it.bad = false;
  start_list<BK, kCache>(it.s0.a, p, u, 0, 0, s_cb, s_ib, s_pb, it.bad);
  start_list<BK, kCache>(it.s0.b, p, u, 0, 1, s_cb, s_ib, s_pb, it.bad);
  start_list<BK, kCache>(it.s1.a, p, u, 1, 0, s_cb, s_ib, s_pb, it.bad);
  start_list<BK, kCache>(it.s1.b, p, u, 1, 1, s_cb, s_ib, s_pb, it.bad);
  return it;
}

// ---------------------------------------------------------------------- the kernel -------------
// kCache: chunked prefill onto a (paged) cache; the plain prefill is compiled separately, with no
// prefix and direct row indexing. kFp8: e4m3 Q and K (QK^T on kind::f8f6f4), bf16 V.
// Paired schedule: a unit runs two query tiles of one kv-head (the design above).
template <int BK, bool kCache, bool kFp8>
__device__ __forceinline__ void attn_pairs(const AttnParams& p) {
  using C = Cfg<BK, kFp8>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kOffQ, sK = sbase + C::kOffK, sV = sbase + C::kOffV;
  const uint32_t bar0 = sbase + C::kOffBar;
  const uint32_t b_q_full = bar0, b_q_empty = bar0 + 8;
  auto b_k_full = [&](int i) { return bar0 + 16 + 8 * i; };
  auto b_k_empty = [&](int i) { return bar0 + 16 + 8 * (C::kStages + i); };
  auto b_v_full = [&](int i) { return bar0 + 16 + 8 * (2 * C::kStages + i); };
  auto b_v_empty = [&](int i) { return bar0 + 16 + 8 * (3 * C::kStages + i); };
  const uint32_t b_s_full0 = bar0 + 16 + 8 * (4 * C::kStages);
  const uint32_t b_p_full0 = b_s_full0 + 16;
  const uint32_t b_o_final0 = b_p_full0 + 16;
  const uint32_t b_drain = b_o_final0 + 16, b_never = b_drain + 8;
  auto b_item = [&](uint32_t x) { return b_never + 8 + 8 * (x % kRing); };
  auto b_item_empty = [&](uint32_t x) { return b_never + 8 + 8 * kRing + 8 * (x % kRing); };
  volatile int* s_item = reinterpret_cast<volatile int*>(smem + C::kOffRing);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int* s_ok = reinterpret_cast<int*>(smem + C::kOffMisc + 8);
  const int S = p.seq.num_seqs;
  int* s_cu = reinterpret_cast<int*>(smem + C::kOffTab);
  int* s_cb = s_cu + (S + 1);
  int* s_ct = s_cb + (S + 1);
  int* s_pb = s_ct + (S + 1);
  int* s_ckb = s_pb + (S + 1);
  long long* s_ib = reinterpret_cast<long long*>(smem + C::kOffTab + 20 * (S + 1) + 4);
  s_ib = reinterpret_cast<long long*>(((uintptr_t)s_ib + 7) & ~(uintptr_t)7);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;

  if (threadIdx.x == 0) {
    mbar_init(b_q_full, 1);
    mbar_init(b_q_empty, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(b_k_full(i), 1);
      mbar_init(b_k_empty(i), 1);
      mbar_init(b_v_full(i), 1);
      mbar_init(b_v_empty(i), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(b_s_full0 + 8 * k, 1);
      mbar_init(b_p_full0 + 8 * k, 128);
      mbar_init(b_o_final0 + 8 * k, 1);
    }
    mbar_init(b_drain, 1);
    mbar_init(b_never, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(b_item(i), 1);
      mbar_init(b_item_empty(i), kRingReaders);
    }
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
  // unit table: Hq units (one per q-head) per 256 query rows (a pair of query tiles)
  const bool ok = build_seq_tables(p.seq, s_cu, s_cb, s_ct, s_ib, p.hq, 2 * kTileM, p.hq, s_ok, p.dev_status,
                                   s_pb, s_ckb) &&
                  (p.dense || s_ib[S] == p.index_elems);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (!ok && threadIdx.x == 0 && !p.dense) dev_flag(p.dev_status, kDevBadProblem);
  const int num_units = ok ? s_ct[S] : 0;

  if (wg == 0) {
    // register budget of the producer / MMA / idle warpgroup (all four warps execute it)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  }
  if (warp == 0) {
    // =========================================================== TMA producer
    if (lane == 0) {
      uint32_t kit = 0, vit = 0;  // loads issued into the K / V rings
      uint32_t xit = 0;           // item-ring entries published
      int uc = 0, q_issued = 0;   // units started / Q loads issued
      bool fail = false;
      bool bad_list = false, bad_page = false;
      // write the next ring entry once every reader has read the one it replaces
      auto publish = [&](int val) -> bool {
        if (xit >= (uint32_t)kRing && !mbar_wait(b_item_empty(xit), ((xit / kRing) - 1) & 1, p.wait_limit_ns))
          return false;
        s_item[xit % kRing] = val;
        mbar_arrive(b_item(xit));
        ++xit;
        return true;
      };
      int t = blockIdx.x;
      for (int k = 0;; ++uc) {
        if (t >= num_units || fail) break;
        const Unit u = decode_unit(t, s_cu, s_cb, s_ct, s_pb, S, p.group);
        if (!publish(t)) { fail = true; break; }
        if (!mbar_wait(b_q_empty, (uc & 1) ^ 1, p.wait_limit_ns)) { fail = true; break; }
        mbar_arrive_expect_tx(b_q_full, C::kQBytes * u.nslot);
        for (int sl = 0; sl < u.nslot; ++sl) {
          const int y = u.seq0 + u.qt[sl] * kTileM;
          tma_load_2d(sQ + sl * C::kQBytes, &p.tm_q, b_q_full, u.h[sl] * kHeadDim, y);
          if constexpr (!kFp8)  // bf16: the second 64 columns are a second slab
            tma_load_2d(sQ + sl * C::kQBytes + C::kSlabQ, &p.tm_q, b_q_full, u.h[sl] * kHeadDim + 64, y);
        }
        ++q_issued;
        KvIter itr = make_iter<BK, kCache>(p, u, s_cb, s_ib, s_pb);
        // V tile of an item: needed only by its PV, issued after the slot's softmax; it is loaded
        // after the NEXT item's K tile, so that a V slot still held by a pending PV never delays
        // the K loads, which the QK MMAs wait for
        auto load_v = [&](long long vy) -> bool {
          const int vs = vit % C::kStages;
          if (!mbar_wait(b_v_empty(vs), ((vit / C::kStages) & 1) ^ 1, p.wait_limit_ns)) return false;
          mbar_arrive_expect_tx(b_v_full(vs), C::kVBytes);
          tma_load_2d(sV + vs * C::kVBytes, &p.tm_v, b_v_full(vs), u.g * kHeadDim, (int32_t)vy);
          tma_load_2d(sV + vs * C::kVBytes + C::kSlabKV, &p.tm_v, b_v_full(vs), u.g * kHeadDim + 64, (int32_t)vy);
          ++vit;
          return true;
        };
        long long vy = -1;  // V row of the previous item, not loaded yet
        int j, mask;
        while (true) {
          bool more = itr.next(j, mask);
          long long y = (long long)u.seq0 + j * BK;  // first K/V row of key block j
          if constexpr (kCache) {  // pages hold whole blocks
            while (more && (y = kv_row(p.seq, s_cu, u.s, j * BK)) < 0) {
              bad_page = true;  // block table outside the cache: the block is skipped
              more = itr.next(j, mask);
            }
          }
          if (!publish(more ? (j << 4) | mask : kItemEnd)) { fail = true; break; }  // the item, or the unit's end
          if (!more) break;
          const int ks = kit % C::kStages;
          if (!mbar_wait(b_k_empty(ks), ((kit / C::kStages) & 1) ^ 1, p.wait_limit_ns)) { fail = true; break; }
          mbar_arrive_expect_tx(b_k_full(ks), C::kKBytes);
          tma_load_2d(sK + ks * C::kKBytes, &p.tm_k, b_k_full(ks), u.g * kHeadDim, (int32_t)y);
          if constexpr (!kFp8)
            tma_load_2d(sK + ks * C::kKBytes + C::kSlabK, &p.tm_k, b_k_full(ks), u.g * kHeadDim + 64, (int32_t)y);
          ++kit;
          if (vy >= 0 && !load_v(vy)) { fail = true; break; }
          vy = y;
          if (*s_abort) { fail = true; break; }
        }
        if (!fail && vy >= 0 && !load_v(vy)) fail = true;  // the unit's last V tile
        bad_list |= itr.bad;
        if (!fail) t = next_unit(p.sched, ++k);
      }
      if (!fail && !publish(kUnitsEnd)) fail = true;
      sched_release(p.sched);
      if (bad_list) dev_flag(p.dev_status, kDevBadList);
      if (bad_page) dev_flag(p.dev_status, kDevBadProblem);
      if (fail) {
        *s_abort = 1;
        dev_flag(p.dev_status, kDevTimeout);
        // let issued copies land before the CTA can exit (own, generous limit: copies always land)
        for (int i = 0; i < C::kStages; ++i) {
          if (kit > (uint32_t)i) mbar_wait(b_k_full(i), ((kit - 1 - i) / C::kStages) & 1, kDrainLimitNs);
          if (vit > (uint32_t)i) mbar_wait(b_v_full(i), ((vit - 1 - i) / C::kStages) & 1, kDrainLimitNs);
        }
        if (q_issued > 0) mbar_wait(b_q_full, (uint32_t)(q_issued - 1) & 1, kDrainLimitNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // =========================================================== tcgen05 issuer
    if (lane == 0) {
      uint32_t kit = 0, vit = 0;  // K / V tiles consumed
      uint32_t cnt[2] = {0, 0};   // items processed per slot (S/P barrier phases)
      int uc = 0;
      bool fail = false;
      // O_k += P_k V for the slot's previous item (V tile vit % kStages)
      auto pv = [&](int k, bool first) -> bool {
        if (!mbar_wait(b_p_full0 + 8 * k, (cnt[k] - 1) & 1, p.wait_limit_ns)) return false;
        const int vs = vit % C::kStages;
        if (!mbar_wait(b_v_full(vs), (vit / C::kStages) & 1, p.wait_limit_ns)) return false;
        tc_fence_after();
        const uint64_t vdesc = sdesc_sw128(sV + vs * C::kVBytes, C::kSlabKV, 1024);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)  // 16 keys = 16 rows of 128 bytes per step
          mma_ts(tmem + tmem_o(k), tmem + tmem_s(k) + kk * 8, desc_advance(vdesc, kk * (2048 >> 4)), C::kIdescPV,
                 (!first || kk > 0) ? 1u : 0u);
        return true;
      };
      // S_k = Q_k K^T for the current item (K tile at kbase)
      auto qk = [&](int k, uint32_t kbase) {
        const uint64_t qdesc = sdesc_sw128(sQ + k * C::kQBytes, 16, 1024);
        const uint64_t kdesc = sdesc_sw128(kbase, 16, 1024);
        if constexpr (kFp8) {
          // 4 steps of 32 e4m3 = 32 bytes inside the single 128-byte swizzle atom
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 32; ++kk)
            mma_ss_f8(tmem + tmem_s(k), desc_advance(qdesc, kk * 2), desc_advance(kdesc, kk * 2), C::kIdescQK,
                      kk > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk) {
            // 16 bf16 = 32 bytes inside the swizzle atom; 64 columns per slab
            const uint32_t qoff = ((kk >> 2) * C::kSlabQ + (kk & 3) * 32) >> 4;
            const uint32_t koff = ((kk >> 2) * C::kSlabK + (kk & 3) * 32) >> 4;
            mma_ss(tmem + tmem_s(k), desc_advance(qdesc, qoff), desc_advance(kdesc, koff), C::kIdescQK,
                   kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(b_s_full0 + 8 * k);
        ++cnt[k];
      };
      uint32_t xit = 0;  // item-ring entries read
      auto read_item = [&](int& e) -> bool {
        if (!mbar_wait(b_item(xit), (xit / kRing) & 1, p.wait_limit_ns)) return false;
        e = s_item[xit % kRing];
        mbar_arrive(b_item_empty(xit));
        ++xit;
        return true;
      };
      for (;; ++uc) {
        int t;
        if (!read_item(t)) { fail = true; break; }
        if (t == kUnitsEnd) break;
        const Unit u = decode_unit(t, s_cu, s_cb, s_ct, s_pb, S, p.group);
        if (!mbar_wait(b_q_full, uc & 1, p.wait_limit_ns)) { fail = true; break; }
        tc_fence_after();
        // Only the slots whose lists hold an item's block take part in it (bits 2k, 2k+1 of its
        // row mask): the others skip its QK, PV and softmax. A slot's PV for item n-1 is issued at
        // item n (before its QK of item n, whose S overwrites P), so V(n-1) is released there.
        int e, n = 0;
        int prev_part = 0;          // slots that took part in the previous item (their PV is due)
        bool had_pv[2] = {false, false};
        if (!read_item(e)) { fail = true; break; }
        bool more = e != kItemEnd;
        while (more) {
          const int mask = e & 15;
          const int part = (((mask & 3) != 0) ? 1 : 0) | (((mask & 12) != 0 && u.nslot == 2) ? 2 : 0);
          const int ks = kit % C::kStages;
          if (!mbar_wait(b_k_full(ks), (kit / C::kStages) & 1, p.wait_limit_ns)) { fail = true; break; }
          tc_fence_after();
          const uint32_t kbase = sK + ks * C::kKBytes;
          // A slot that had no part in the previous item issued its last PV earlier: its QK goes
          // first, so that it does not wait for the other slot's softmax (single-slot items of
          // alternating slots then overlap like shared ones). A slot that took part issues the
          // previous item's PV before this item's QK (S_k(n) overwrites P_k(n-1)).
if (part == 3 && prev_part == 3) {
            // both slots in both items (every item at density 1): the pingpong order PV0 QK0 PV1 QK1
            if (!pv(0, !had_pv[0])) { fail = true; break; }
            had_pv[0] = true;
            qk(0, kbase);
            if (!pv(1, !had_pv[1])) { fail = true; break; }
            had_pv[1] = true;
            qk(1, kbase);
          } else {
  #pragma unroll
            for (int sl = 0; sl < 2; ++sl)
              if (((part & ~prev_part) >> sl) & 1) qk(sl, kbase);
  #pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
              if ((prev_part >> sl) & 1) {
                if (!pv(sl, !had_pv[sl])) { fail = true; break; }
                had_pv[sl] = true;
                if ((part >> sl) & 1) qk(sl, kbase);
              }
            }
          }
          if (fail) break;
          if (n > 0) {  // the previous item's PVs are issued: release its V tile
            mma_commit(b_v_empty(vit % C::kStages));
            ++vit;
          }
          mma_commit(b_k_empty(ks));
          ++kit;
          prev_part = part;
          if (!read_item(e)) { fail = true; break; }
          more = e != kItemEnd;
          if (!more) mma_commit(b_q_empty);
          ++n;
          if (*s_abort) { fail = true; break; }
        }
        if (fail) break;
        if (n > 0) {
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            if ((prev_part >> sl) & 1) {
              if (!pv(sl, !had_pv[sl])) { fail = true; break; }
              had_pv[sl] = true;
            }
          }
          if (fail) break;
          mma_commit(b_v_empty(vit % C::kStages));
          ++vit;
          if (had_pv[0]) mma_commit(b_o_final0);
          if (had_pv[1]) mma_commit(b_o_final0 + 8);
        } else {
          mma_commit(b_q_empty);  // empty kv list: release Q without touching O
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
  } else if (wg >= 1) {
    // =========================================================== softmax / correction / epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int slot = wg - 1;
    const int q4 = warp & 3;                  // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;             // row of the slot's tile owned by this thread
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int half = (BK == 64) ? (r >> 6) : 0;
    const int mbit = 2 * slot + half;         // this row's bit in the iteration mask
    const uint32_t s_col = tmem + lane_off + tmem_s(slot), o_col = tmem + lane_off + tmem_o(slot);
    const uint32_t b_s_full = b_s_full0 + 8 * slot, b_p_full = b_p_full0 + 8 * slot;
    const uint32_t b_o_final = b_o_final0 + 8 * slot;
    uint32_t cnt = 0;  // items processed by this slot (S/P barrier phases)
    uint32_t xit = 0;  // item-ring entries read
    int fc = 0;        // units of this slot with a non-empty list (o_final phases)
    bool fail = false;
    if (p.test_unsignalled_wait && num_units > 0)
      fail = __any_sync(kFull, !mbar_wait(b_never, 0, p.wait_limit_ns));
    // the next ring entry (warp-collective; lane 0 releases the entry once the whole warp has read it)
    auto read_entry = [&](int& e) -> bool {
      if (__any_sync(kFull, !mbar_wait(b_item(xit), (xit / kRing) & 1, p.wait_limit_ns))) return false;
      e = s_item[xit % kRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(b_item_empty(xit));
      ++xit;
      return true;
    };
    while (!fail) {
      int t;
      if (!read_entry(t)) { fail = true; break; }
      if (t == kUnitsEnd) break;
      const Unit u = decode_unit(t, s_cu, s_cb, s_ct, s_pb, S, p.group);
      const bool active = slot < u.nslot;     // an idle slot only consumes the unit's ring entries
      const int qpos = u.qt[slot] * kTileM + r;  // local query position of this row
      // Rows past the sequence end (the last tile's padding) hold whatever follows in memory: they
      // never take part in the warp's path votes, so a sequence's outputs do not depend on its
      // neighbours in the batch (or on what lies past the end of a cache page).
      const bool pad = qpos >= u.len;
      // FP8 with per-block scales: this row's softmax scale times its query block's 2^q_exp; each item
      // multiplies in its key block's 2^k_exp (plain prefill only: key block j is global block gb0 + j)
      float row_sl2 = p.scale_log2;
      if constexpr (kFp8) {
        const int qblk = u.qt[slot] * (kTileM / BK) + half;
        if (p.q_exp && active && qblk < u.nb) row_sl2 = p.scale_log2 * pow2i(__ldg(p.q_exp + (long long)(u.gb0 + qblk) * p.hq + u.h[slot]));
      }
      float m_run = -INFINITY, l_run = 0.f;
      int n = 0;
      while (true) {
        int e;
        if (!read_entry(e)) { fail = true; break; }
        if (e == kItemEnd) break;
        if (!active) continue;
        const int j = e >> 4, mask = e & 15;
        if (((mask >> (2 * slot)) & 3) == 0) continue;  // no list of this slot holds block j
        int kexp = 0;
        if constexpr (kFp8)
          if (p.k_exp) kexp = __ldg(p.k_exp + (long long)(u.gb0 + j) * p.hkv + u.g);  // lands during the S wait
        // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform
        if (__any_sync(kFull, !mbar_wait(b_s_full, cnt & 1, p.wait_limit_ns))) { fail = true; break; }
        tc_fence_after();
        // causal mask (diagonal tiles) and the list mask of this row's query block
        const int valid = ((mask >> mbit) & 1) ? (qpos - (j - (kCache ? u.pb : 0)) * BK) : -1;
        const bool masked = valid < BK - 1;
        float sl2 = row_sl2;  // this item's logits in log2 units per unit of S
        if constexpr (kFp8)
          if (p.k_exp) sl2 = row_sl2 * pow2i(kexp);
        const uint64_t scale2 = f2_make(sl2, sl2);
        uint32_t pk[BK / 2];
        // Fast path, for unmasked items once the row has a reference max: no max pass. S streams
        // from TMEM in 32-column chunks (the next chunk loads while this one is exponentiated)
        // against the current reference max, and the item's row sum decides afterwards: a sum of
        // at most 2^16 bounds every P below 2^16 (finite, and exact in the shared scale), so the
        // item stands without a rescale. A larger (or non-finite) sum sends the warp through the
        // exact path below, which reloads S (still in TMEM: P is stored only at the end).
        bool done = false;
        if (__all_sync(kFull, pad || (!masked && m_run != -INFINITY))) {
          const uint64_t negm2 = f2_make(-m_run, -m_run);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
          uint32_t cb[2][32];
          tmem_ld32(s_col, cb[0]);
#pragma unroll
          for (int c = 0; c < BK / 32; ++c) {
            tmem_wait_ld();
            reg_fence32(cb[c & 1]);
            if (c + 1 < BK / 32) tmem_ld32(s_col + 32 * (c + 1), cb[(c + 1) & 1]);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int pr = 16 * c + e / 2;  // pair index within the item
              const uint64_t x2 = ffma2(f2_bits(cb[c & 1][e], cb[c & 1][e + 1]), scale2, negm2);
              float x0, x1;
              f2_split(x2, x0, x1);
              const uint64_t p2 = f2_make(ex2_approx(x0), ex2_approx(x1));
              acc[pr & 3] = fadd2(acc[pr & 3], p2);
              float p0, p1;
              f2_split(p2, p0, p1);
              pk[pr] = pack_bf16x2(p0, p1);
            }
          }
          float a0, a1, b0, b1;
          f2_split(fadd2(acc[0], acc[1]), a0, a1);
          f2_split(fadd2(acc[2], acc[3]), b0, b1);
          const float isum = (a0 + a1) + (b0 + b1);
          done = __all_sync(kFull, pad || isum <= kFastSumLimit);
          if (done) l_run += isum;
        }
        if (!done) {
          uint32_t sr[BK];
#pragma unroll
          for (int c = 0; c < BK; c += 32)
            tmem_ld32(s_col + c, *reinterpret_cast<uint32_t(*)[32]>(&sr[c]));
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < BK; c += 32) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[c]));
          float mx;
          {
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            // keys past the row's causal limit (every key when its list lacks the block) become -inf
            // here, and exact zeros below (MUFU ex2(-inf) = 0); one loop for masked and unmasked items
            // keeps the kernel's code short (instruction-cache misses show in its stall profile)
#pragma unroll
            for (int c = 0; c < BK; c += 8) {
#pragma unroll
              for (int a = 0; a < 4; ++a) {
                const float v0 = (c + 2 * a <= valid) ? __uint_as_float(sr[c + 2 * a]) : -INFINITY;
                const float v1 = (c + 2 * a + 1 <= valid) ? __uint_as_float(sr[c + 2 * a + 1]) : -INFINITY;
                sr[c + 2 * a] = __float_as_uint(v0);
                sr[c + 2 * a + 1] = __float_as_uint(v1);
                m4[a] = fmax3(m4[a], v0, v1);
              }
            }
            mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
          }
          const float m_new = fmaxf(m_run, mx * sl2);
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
            // S_k(n) was committed after PV_k(n-1): O_k is complete; lanes that did not grow scale by 1
            const uint64_t a2 = f2_make(alpha, alpha);
#pragma unroll 1
            for (int c = 0; c < kHeadDim; c += 32) {
              uint32_t o[32];
              tmem_ld32(o_col + c, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float lo, hi;
                f2_split(fmul2(f2_bits(o[e], o[e + 1]), a2), lo, hi);
                o[e] = __float_as_uint(lo);
                o[e + 1] = __float_as_uint(hi);
              }
              tmem_st32(o_col + c, o);
            }
          }
          const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
          const uint64_t negm2 = f2_make(-m_use, -m_use);
          uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < BK; c += 2) {
            const uint64_t x2 = ffma2(f2_bits(sr[c], sr[c + 1]), scale2, negm2);
            float x0, x1;
            f2_split(x2, x0, x1);
            const uint64_t p2 = f2_make(ex2_approx(x0), ex2_approx(x1));
            sum2[(c >> 1) & 1] = fadd2(sum2[(c >> 1) & 1], p2);
            float p0, p1;
            f2_split(p2, p0, p1);
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
          float a0, a1, b0, b1;
          f2_split(sum2[0], a0, a1);
          f2_split(sum2[1], b0, b1);
          l_run += (a0 + a1) + (b0 + b1);
        }
#pragma unroll
        for (int c = 0; c < BK / 2; c += 32)
          tmem_st32(s_col + c, *reinterpret_cast<uint32_t(*)[32]>(&pk[c]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p_full);
        ++cnt;
        ++n;
      }
      if (__any_sync(kFull, fail || *s_abort)) { fail = true; break; }
      if (!active) continue;
      const bool row_ok = qpos < u.len;
      const long long row = (long long)u.seq0 + qpos;
      if (n == 0) {  // empty kv list (malformed input): zero output, LSE -inf
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (row * p.hq + u.h[slot]) * kHeadDim);
          for (int c = 0; c < kHeadDim / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[(long long)u.h[slot] * p.seq.total_tokens + row] = -INFINITY;
        }
        continue;
      }
      // ---- epilogue: O / l -> bf16, LSE
      if (__any_sync(kFull, !mbar_wait(b_o_final, fc & 1, p.wait_limit_ns))) { fail = true; break; }
      ++fc;
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      uint16_t* orow = p.out + (row * p.hq + u.h[slot]) * kHeadDim;
#pragma unroll 1
      for (int c = 0; c < kHeadDim; c += 32) {
        uint32_t o[32];
        tmem_ld32(o_col + c, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
        if (row_ok) {
          if (p.out32) {  // 32-byte stores: a whole sector per thread and half the store instructions
            st_global_v8(orow + c, w);
            st_global_v8(orow + c + 16, w + 8);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
            dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
          }
        }
      }
      if (row_ok && p.lse) {
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        p.lse[(long long)u.h[slot] * p.seq.total_tokens + row] =
            l_run > 0.f ? (m_use + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      }
      tc_fence_before();
    }
    if (fail) {
      *s_abort = 1;
      dev_flag(p.dev_status, kDevTimeout);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ======================================================================= row schedule ============
// Row schedule (plain bf16 prefill, B = 128), for sparse lists: a unit is one query tile (128 rows of
// one q-head); both softmax warpgroups split every item's 128 keys (warpgroup 1 keys 0..63, warpgroup
// 2 keys 64..127, each thread one row of its half) and the two TMEM S buffers alternate between
// consecutive items, so QK(n+1) runs during softmax(n). Nothing depends on a partner row, so lists of
// any lengths keep the pipeline full; the price is K/V tiles loaded once per row (no sharing between
// two rows), which makes it slower than the paired schedule when most blocks are kept (measured at
// 128K: 23% slower at density 1, 9% at 0.46, 12% faster at 0.06; at 32K 5% faster at 0.32).
// Each half keeps its own running max, row sum and accumulator (O0 = P0 V[0, 64), O1 = P1 V[64,
// 128)), so the halves never wait for each other inside a unit; the epilogue exchanges (max, sum)
// once and writes (a0 O0 + a1 O1) / (a0 l0 + a1 l1) with a_h = 2^(m_h - max(m0, m1)).
// TMEM: S0 | S1 | O0 | O1 (128 columns each). P of an item overwrites the S columns its own half
// has read: keys 0..63 packed into columns 0..31, keys 64..127 into columns 96..127.
namespace rows {
constexpr int kQBufs = 2, kKStages = 2, kVStages = 2;  // Q tiles, K ring, V ring
constexpr uint32_t kQBytes = kTileM * kHeadDim * 2, kKBytes = 128 * kHeadDim * 2, kVBytes = kKBytes;
constexpr uint32_t kSlab = 128 * 128;  // 128 rows x 128 bytes
constexpr uint32_t kOffQ = 0, kOffK = kQBufs * kQBytes, kOffV = kOffK + kKStages * kKBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kVBytes;
// q_full[2], q_empty[2], k_full[], v_full[], v_empty[], s_full[2], p_full[2], o_final, drain,
// item[kRing], item_empty[kRing], pair[4] (the two softmax warps of one 32-row quarter exchange row
// statistics: 64 arrivals per phase, bounded waits), never (test hook).
// A K stage is released by the S barrier of the QK that read it (K stage n % 2 = S buffer n % 2),
// and an O rescale waits for the previous item's PV on that PV's V-empty barrier: two commits per
// item fewer for the issuing thread. Neither wait can alias a later phase: the next phase of either
// barrier needs a tile or a P that the waiter has not produced yet.
static_assert(kKStages == 2, "K stages are released through the two S buffers' barriers");
constexpr int kNumBars = 4 + kKStages + 2 * kVStages + 4 + 2 + 2 * kRing + 4 + 1;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;          // tmem base, abort, ok
constexpr uint32_t kOffRing = kOffMisc + 16;
constexpr uint32_t kOffX = kOffRing + 4 * kRing;               // exchange: float max[2 half][128], sum[2 half][128]
constexpr uint32_t kXBytes = 2 * 2 * 128 * 4 + 2 * 2 * 4 * 4;
constexpr uint32_t kOffTab = (kOffX + kXBytes + 15) & ~15u;
constexpr uint32_t smem_bytes(int num_seqs) { return kOffTab + 5 * 4 * (num_seqs + 1) + 8 * (num_seqs + 1) + 16 + 1024; }
constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kHeadDim, 0, 1);
}  // namespace rows

__device__ __forceinline__ void attn_rows(const AttnParams& p) {
  using namespace rows;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV;
  const uint32_t bar0 = sbase + kOffBar;
  auto b_q_full = [&](int i) { return bar0 + 8 * i; };
  auto b_q_empty = [&](int i) { return bar0 + 16 + 8 * i; };
  auto b_k_full = [&](int i) { return bar0 + 32 + 8 * i; };
  auto b_v_full = [&](int i) { return bar0 + 32 + 8 * (kKStages + i); };
  auto b_v_empty = [&](int i) { return bar0 + 32 + 8 * (kKStages + kVStages + i); };
  const uint32_t b_s_full0 = bar0 + 32 + 8 * (kKStages + 2 * kVStages), b_p_full0 = b_s_full0 + 16;
  const uint32_t b_o_final = b_p_full0 + 16, b_drain = b_o_final + 8;
  auto b_item = [&](uint32_t x) { return b_drain + 8 + 8 * (x % kRing); };
  auto b_item_empty = [&](uint32_t x) { return b_drain + 8 + 8 * kRing + 8 * (x % kRing); };
  auto b_pair = [&](int q) { return b_drain + 8 + 16 * kRing + 8 * q; };
  const uint32_t b_never = b_drain + 8 + 16 * kRing + 32;
  volatile int* s_item = reinterpret_cast<volatile int*>(smem + kOffRing);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  int* s_ok = reinterpret_cast<int*>(smem + kOffMisc + 8);
  volatile float* s_xf = reinterpret_cast<volatile float*>(smem + kOffX);             // [par][half][row]
  const int S = p.seq.num_seqs;
  int* s_cu = reinterpret_cast<int*>(smem + kOffTab);
  int* s_cb = s_cu + (S + 1);
  int* s_ct = s_cb + (S + 1);
  int* s_pb = s_ct + (S + 1);
  int* s_ckb = s_pb + (S + 1);
  long long* s_ib = reinterpret_cast<long long*>(smem + kOffTab + 20 * (S + 1) + 4);
  s_ib = reinterpret_cast<long long*>(((uintptr_t)s_ib + 7) & ~(uintptr_t)7);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(b_q_full(i), 1);
      mbar_init(b_q_empty(i), 1);
      mbar_init(b_s_full0 + 8 * i, 1);
      mbar_init(b_p_full0 + 8 * i, 256);
    }
    for (int i = 0; i < kKStages; ++i) mbar_init(b_k_full(i), 1);
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(b_v_full(i), 1);
      mbar_init(b_v_empty(i), 1);
    }
    mbar_init(b_o_final, 1);
    mbar_init(b_drain, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(b_item(i), 1);
      mbar_init(b_item_empty(i), kRingReaders);
    }
    for (int i = 0; i < 4; ++i) mbar_init(b_pair(i), 64);
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
  // unit table: Hq units (one per q-head) per 128 query rows
  const bool ok = build_seq_tables(p.seq, s_cu, s_cb, s_ct, s_ib, p.hq, kTileM, p.hq, s_ok, p.dev_status, s_pb, s_ckb) &&
                  (p.dense || s_ib[S] == p.index_elems);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (!ok && threadIdx.x == 0 && !p.dense) dev_flag(p.dev_status, kDevBadProblem);
  const int num_units = ok ? s_ct[S] : 0;
  // unit t -> (sequence, kv-head outermost, descending query tile, q-head)
  auto decode1 = [&](int t, int& s, int& g, int& h, int& qt) {
    s = find_seq(s_ct, S, t);
    const int local = t - s_ct[s];
    const int len = s_cu[s + 1] - s_cu[s];
    const int ntile = (len + kTileM - 1) / kTileM;
    const int per_g = ntile * p.group;
    g = local / per_g;
    const int rem = local % per_g;
    qt = ntile - 1 - rem / p.group;
    h = g * p.group + rem % p.group;
  };
  if (wg == 0) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));

  if (warp == 0) {
    // =========================================================== producer
    if (lane == 0) {
      uint32_t kit = 0, vit = 0, xit = 0;
      int uc = 0;
      bool fail = false, bad = false;
      auto publish = [&](int val) -> bool {
        if (xit >= (uint32_t)kRing && !mbar_wait(b_item_empty(xit), ((xit / kRing) - 1) & 1, p.wait_limit_ns)) return false;
        s_item[xit % kRing] = val;
        mbar_arrive(b_item(xit));
        ++xit;
        return true;
      };
      int t = blockIdx.x;
      for (int k = 0;; ++uc) {
        if (t >= num_units || fail) break;
        int s, g, h, qt;
        decode1(t, s, g, h, qt);
        const int seq0 = s_cu[s], nb = s_cb[s + 1] - s_cb[s];
        if (!publish(t)) { fail = true; break; }
        const int qs = uc % kQBufs;
        if (!mbar_wait(b_q_empty(qs), ((uc / kQBufs) & 1) ^ 1, p.wait_limit_ns)) { fail = true; break; }
        mbar_arrive_expect_tx(b_q_full(qs), kQBytes);
        tma_load_2d(sQ + qs * kQBytes, &p.tm_q, b_q_full(qs), h * kHeadDim, seq0 + qt * kTileM);
        tma_load_2d(sQ + qs * kQBytes + kSlab, &p.tm_q, b_q_full(qs), h * kHeadDim + 64, seq0 + qt * kTileM);
        // the row's list (B = 128: one query block per tile)
        const int blk = qt;
        const int jd = blk;
        int n = 0;
        const int32_t* list = nullptr;
        if (blk < nb) {
          if (p.dense) n = jd + 1;
          else {
            list = p.indices + list_row(s_cb, s_ib, s_pb, s, h, blk);
            n = min(max(__ldg(p.counts + (long long)h * p.seq.total_blocks + s_cb[s] + blk), 0), jd + 1);
          }
        }
        long long vy = -1;
        auto load_v = [&](long long y) -> bool {
          const int vs = vit % kVStages;
          if (!mbar_wait(b_v_empty(vs), ((vit / kVStages) & 1) ^ 1, p.wait_limit_ns)) return false;
          mbar_arrive_expect_tx(b_v_full(vs), kVBytes);
          tma_load_2d(sV + vs * kVBytes, &p.tm_v, b_v_full(vs), g * kHeadDim, (int32_t)y);
          tma_load_2d(sV + vs * kVBytes + kSlab, &p.tm_v, b_v_full(vs), g * kHeadDim + 64, (int32_t)y);
          ++vit;
          return true;
        };
        for (int i = 0; i < n; ++i) {
          const int j = p.dense ? i : __ldg(list + i);
          if (j < 0 || j > jd) { bad = true; continue; }
          const long long y = (long long)seq0 + (long long)j * 128;
          if (!publish(j)) { fail = true; break; }
          const int ks = kit % kKStages;
          // stage ks is free once QK(kit - 2), which read it, is done (S buffer ks, that QK's phase)
          if (kit >= (uint32_t)kKStages &&
              !mbar_wait(b_s_full0 + 8 * ks, ((kit - kKStages) / 2) & 1, p.wait_limit_ns)) { fail = true; break; }
          mbar_arrive_expect_tx(b_k_full(ks), kKBytes);
          tma_load_2d(sK + ks * kKBytes, &p.tm_k, b_k_full(ks), g * kHeadDim, (int32_t)y);
          tma_load_2d(sK + ks * kKBytes + kSlab, &p.tm_k, b_k_full(ks), g * kHeadDim + 64, (int32_t)y);
          ++kit;
          if (vy >= 0 && !load_v(vy)) { fail = true; break; }
          vy = y;
          if (*s_abort) { fail = true; break; }
        }
        if (!fail && vy >= 0 && !load_v(vy)) fail = true;
        if (!fail && !publish(kItemEnd)) fail = true;
        if (!fail) t = next_unit(p.sched, ++k);
      }
      if (!fail && !publish(kUnitsEnd)) fail = true;
      sched_release(p.sched);
      if (bad) dev_flag(p.dev_status, kDevBadList);
      if (fail) {
        *s_abort = 1;
        dev_flag(p.dev_status, kDevTimeout);
        for (int i = 0; i < kKStages; ++i)
          if (kit > (uint32_t)i) mbar_wait(b_k_full(i), ((kit - 1 - i) / kKStages) & 1, kDrainLimitNs);
        for (int i = 0; i < kVStages; ++i)
          if (vit > (uint32_t)i) mbar_wait(b_v_full(i), ((vit - 1 - i) / kVStages) & 1, kDrainLimitNs);
        for (int i = 0; i < kQBufs && i < uc + 1; ++i) {
          const int u_last = uc - i;
          if (u_last >= 0) mbar_wait(b_q_full(u_last % kQBufs), (u_last / kQBufs) & 1, kDrainLimitNs);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // =========================================================== MMA issuer
    if (lane == 0) {
      uint32_t kit = 0, vit = 0, xit = 0;
      uint32_t g_it = 0;  // items issued so far (S buffer g_it % 2; phase (g_it / 2) & 1)
      int uc = 0;
      bool fail = false;
      auto read_item = [&](int& e) -> bool {
        if (!mbar_wait(b_item(xit), (xit / kRing) & 1, p.wait_limit_ns)) return false;
        e = s_item[xit % kRing];
        mbar_arrive(b_item_empty(xit));
        ++xit;
        return true;
      };
      auto qk = [&](uint32_t qbase, uint32_t kbase, uint32_t buf) {
        const uint64_t qdesc = sdesc_sw128(qbase, 16, 1024), kdesc = sdesc_sw128(kbase, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kSlab + (kk & 3) * 32) >> 4;
          mma_ss(tmem + 128u * buf, desc_advance(qdesc, off), desc_advance(kdesc, off), kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(b_s_full0 + 8 * buf);
      };
      // O0 += P0 V[0, 64) and O1 += P1 V[64, 128) of global item gi (P in S buffer gi % 2: keys
      // 0..63 packed in columns 0..31, keys 64..127 in columns 96..127), V tile vit % kVStages
      auto pv = [&](uint32_t gi, bool first) -> bool {
        const uint32_t buf = gi & 1;
        if (!mbar_wait(b_p_full0 + 8 * buf, (gi >> 1) & 1, p.wait_limit_ns)) return false;
        const int vs = vit % kVStages;
        if (!mbar_wait(b_v_full(vs), (vit / kVStages) & 1, p.wait_limit_ns)) return false;
        tc_fence_after();
        const uint64_t vdesc = sdesc_sw128(sV + vs * kVBytes, kSlab, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bdesc = desc_advance(vdesc, kk * (2048 >> 4));
          const uint32_t acol = 128u * buf + (kk < 4 ? 8u * kk : 96u + 8u * (kk - 4));
          mma_ts(tmem + (kk < 4 ? 256u : 384u), tmem + acol, bdesc, kIdescPV, (!first || (kk & 3) > 0) ? 1u : 0u);
        }
        mma_commit(b_v_empty(vs));
        ++vit;
        return true;
      };
      for (;; ++uc) {
        int t;
        if (!read_item(t)) { fail = true; break; }
        if (t == kUnitsEnd) break;
        const int qs = uc % kQBufs;
        if (!mbar_wait(b_q_full(qs), (uc / kQBufs) & 1, p.wait_limit_ns)) { fail = true; break; }
        tc_fence_after();
        const uint32_t qbase = sQ + qs * kQBytes;
        int e, n = 0;
        if (!read_item(e)) { fail = true; break; }
        while (e != kItemEnd) {
          const int ks = kit % kKStages;
          if (!mbar_wait(b_k_full(ks), (kit / kKStages) & 1, p.wait_limit_ns)) { fail = true; break; }
          tc_fence_after();
          qk(qbase, sK + ks * kKBytes, g_it & 1);   // S(n): buffer free since PV(n-2) was issued
          ++kit;
          if (n > 0 && !pv(g_it - 1, n == 1)) { fail = true; break; }  // PV(n-1) once its P is stored
          ++g_it;
          ++n;
          if (!read_item(e)) { fail = true; break; }
          if (e == kItemEnd) mma_commit(b_q_empty(qs));
          if (*s_abort) { fail = true; break; }
        }
        if (fail) break;
        if (n > 0) {
          if (!pv(g_it - 1, n == 1)) { fail = true; break; }
          mma_commit(b_o_final);
        } else {
          mma_commit(b_q_empty(qs));
        }
      }
      if (fail) {
        *s_abort = 1;
        dev_flag(p.dev_status, kDevTimeout);
      }
      mma_commit(b_drain);
      mbar_wait(b_drain, 0, kDrainLimitNs);
    }
    __syncwarp();
  } else if (wg >= 1) {
    // =========================================================== softmax (one half of every item's keys)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int hf = wg - 1;                    // key half
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t o_col = tmem + lane_off + 256u + 128u * hf;  // this half's own O (all 128 columns)
    uint32_t g_it = 0;                        // items processed (global, buffer parity)
    uint32_t xit = 0;
    int fc = 0;
    bool fail = false;
    uint32_t pcnt = 0;  // pair exchanges so far (pair barrier phases)
    auto pair_sync = [&]() -> bool {
      mbar_arrive(b_pair(q4));
      const bool okk = !__any_sync(kFull, !mbar_wait(b_pair(q4), pcnt & 1, p.wait_limit_ns));
      ++pcnt;
      return okk;
    };
    if (p.test_unsignalled_wait && num_units > 0)
      fail = __any_sync(kFull, !mbar_wait(b_never, 0, p.wait_limit_ns));
    auto read_entry = [&](int& e) -> bool {
      if (__any_sync(kFull, !mbar_wait(b_item(xit), (xit / kRing) & 1, p.wait_limit_ns))) return false;
      e = s_item[xit % kRing];
      __syncwarp();
      if (lane == 0) mbar_arrive(b_item_empty(xit));
      ++xit;
      return true;
    };
    while (!fail) {
      int t;
      if (!read_entry(t)) { fail = true; break; }
      if (t == kUnitsEnd) break;
      int s, g, h, qt;
      decode1(t, s, g, h, qt);
      const int len = s_cu[s + 1] - s_cu[s];
      const int qpos = qt * kTileM + r;
      const bool pad = qpos >= len;
      float m_run = -INFINITY, l_half = 0.f;
      int n = 0;
      while (true) {
        int e;
        if (!read_entry(e)) { fail = true; break; }
        if (e == kItemEnd) break;
        const int j = e;
        const uint32_t buf = g_it & 1;
        const uint32_t par = (g_it >> 1) & 1;
        if (__any_sync(kFull, !mbar_wait(b_s_full0 + 8 * buf, par, p.wait_limit_ns))) { fail = true; break; }
        tc_fence_after();
        const uint32_t s_col = tmem + lane_off + 128u * buf + 64u * hf;
        const int valid = qpos - j * 128 - 64 * hf;  // my keys 64 hf + c are causal iff c <= valid
        const bool masked = valid < 63;              // some key of my half is masked for this row
        const float sl2 = p.scale_log2;
        const uint64_t scale2 = f2_make(sl2, sl2);
        uint32_t pk[32];
        bool done = false;
        if (__all_sync(kFull, pad || (!masked && m_run != -INFINITY))) {
          const uint64_t negm2 = f2_make(-m_run, -m_run);
          uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
          uint32_t cb[2][32];
          tmem_ld32(s_col, cb[0]);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tmem_wait_ld();
            reg_fence32(cb[c & 1]);
            if (c == 0) tmem_ld32(s_col + 32, cb[1]);
#pragma unroll
            for (int e2 = 0; e2 < 32; e2 += 2) {
              const int pr = 16 * c + e2 / 2;
              const uint64_t x2 = ffma2(f2_bits(cb[c][e2], cb[c][e2 + 1]), scale2, negm2);
              float x0, x1;
              f2_split(x2, x0, x1);
              const uint64_t p2 = f2_make(ex2_approx(x0), ex2_approx(x1));
              acc[pr & 3] = fadd2(acc[pr & 3], p2);
              float p0, p1;
              f2_split(p2, p0, p1);
              pk[pr] = pack_bf16x2(p0, p1);
            }
          }
          float a0, a1, b0, b1;
          f2_split(fadd2(acc[0], acc[1]), a0, a1);
          f2_split(fadd2(acc[2], acc[3]), b0, b1);
          const float hsum = (a0 + a1) + (b0 + b1);
          done = __all_sync(kFull, pad || hsum <= 32768.f);
          if (done) l_half += hsum;
        }
        if (!done) {
          uint32_t sr[64];
          tmem_ld32(s_col, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_wait_ld();
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
#pragma unroll
            for (int a = 0; a < 4; ++a) {
              const float v0 = (c + 2 * a <= valid) ? __uint_as_float(sr[c + 2 * a]) : -INFINITY;
              const float v1 = (c + 2 * a + 1 <= valid) ? __uint_as_float(sr[c + 2 * a + 1]) : -INFINITY;
              sr[c + 2 * a] = __float_as_uint(v0);
              sr[c + 2 * a + 1] = __float_as_uint(v1);
              m4[a] = fmax3(m4[a], v0, v1);
            }
          }
          const float hmax = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
          const float m_new = fmaxf(m_run, hmax * sl2);
          const bool grow = m_new > m_run + 8.0f;
          float alpha = 1.f;
          if (grow) {
            alpha = ex2_approx(m_run - m_new);
            m_run = m_new;
          }
          l_half *= alpha;
          if (n > 0 && __any_sync(kFull, grow)) {
            // O must hold PV(n-1): S(n) was committed after PV(n-2) only; PV(n-1) releases V stage
            // (n-1) % kVStages
            if (__any_sync(kFull, !mbar_wait(b_v_empty((g_it - 1) % kVStages), ((g_it - 1) / kVStages) & 1,
                                             p.wait_limit_ns))) { fail = true; break; }
            tc_fence_after();
            const uint64_t a2 = f2_make(alpha, alpha);
#pragma unroll 1
            for (int c = 0; c < 128; c += 32) {
              uint32_t o[32];
              tmem_ld32(o_col + c, o);
              tmem_wait_ld();
              reg_fence32(o);
#pragma unroll
              for (int e2 = 0; e2 < 32; e2 += 2) {
                float lo, hi;
                f2_split(fmul2(f2_bits(o[e2], o[e2 + 1]), a2), lo, hi);
                o[e2] = __float_as_uint(lo);
                o[e2 + 1] = __float_as_uint(hi);
              }
              tmem_st32(o_col + c, o);
            }
          }
          const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
          const uint64_t negm2 = f2_make(-m_use, -m_use);
          uint64_t sum2[2] = {0ull, 0ull};
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const uint64_t x2 = ffma2(f2_bits(sr[c], sr[c + 1]), scale2, negm2);
            float x0, x1;
            f2_split(x2, x0, x1);
            const uint64_t p2 = f2_make(ex2_approx(x0), ex2_approx(x1));
            sum2[(c >> 1) & 1] = fadd2(sum2[(c >> 1) & 1], p2);
            float p0, p1;
            f2_split(p2, p0, p1);
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
          float a0, a1, b0, b1;
          f2_split(sum2[0], a0, a1);
          f2_split(sum2[1], b0, b1);
          l_half += (a0 + a1) + (b0 + b1);
        }
        tmem_st32(tmem + lane_off + 128u * buf + (hf ? 96u : 0u), pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p_full0 + 8 * buf);
        ++g_it;
        ++n;
      }
      if (__any_sync(kFull, fail || *s_abort)) { fail = true; break; }
      const bool row_ok = !pad;
      const long long row = (long long)s_cu[s] + qpos;
      // the row's statistics: each half's running max and sum (both relative to its own max)
      s_xf[hf * 128 + r] = m_run;
      s_xf[256 + hf * 128 + r] = l_half;
      if (!pair_sync()) { fail = true; break; }
      const float m_oth = s_xf[(1 - hf) * 128 + r], l_oth = s_xf[256 + (1 - hf) * 128 + r];
      if (!pair_sync()) { fail = true; break; }  // both read before the exchange area is reused
      const float m_row = fmaxf(m_run, m_oth);
      const float m_use = (m_row == -INFINITY) ? 0.f : m_row;
      const float a_me = ex2_approx(m_run - m_use), a_oth = ex2_approx(m_oth - m_use);  // 0 for an empty half
      const float l_run = l_half * a_me + l_oth * a_oth;
      if (n == 0) {
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (row * p.hq + h) * kHeadDim + 64 * hf);
          for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          if (p.lse && hf == 0) p.lse[(long long)h * p.seq.total_tokens + row] = -INFINITY;
        }
        continue;
      }
      if (__any_sync(kFull, !mbar_wait(b_o_final, fc & 1, p.wait_limit_ns))) { fail = true; break; }
      ++fc;
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
      // output columns 64 hf .. 64 hf + 63: O0 and O1 there, each weighted by its half's factor
      const float w0 = (hf == 0 ? a_me : a_oth) * inv_l, w1 = (hf == 0 ? a_oth : a_me) * inv_l;
      const uint32_t o0_col = tmem + lane_off + 256u + 64u * hf;
      uint16_t* orow = p.out + (row * p.hq + h) * kHeadDim + 64 * hf;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        uint32_t o[32], o1[32];
        tmem_ld32(o0_col + c, o);
        tmem_ld32(o0_col + 128u + c, o1);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2)
          w[e2] = pack_bf16x2(fmaf(__uint_as_float(o[2 * e2]), w0, __uint_as_float(o1[2 * e2]) * w1),
                              fmaf(__uint_as_float(o[2 * e2 + 1]), w0, __uint_as_float(o1[2 * e2 + 1]) * w1));
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          dst[2] = make_uint4(w[8], w[9], w[10], w[11]);
          dst[3] = make_uint4(w[12], w[13], w[14], w[15]);
        }
      }
      if (row_ok && p.lse && hf == 0)
        p.lse[(long long)h * p.seq.total_tokens + row] =
            l_run > 0.f ? (m_use + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
    }
    if (fail) {
      *s_abort = 1;
      dev_flag(p.dev_status, kDevTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// Schedule choice (plain bf16 prefill, B = 128): the row schedule when fewer than 40% of the causal
// blocks are kept. Every CTA of both kernels sums the list counts (4 bytes per list) before it starts,
// so both take the same decision; p.units forces either schedule. Call with every thread of the CTA.
__device__ __forceinline__ bool rows_chosen(const AttnParams& p) {
  if (p.units != 0) return p.units == 2;
  if (p.dense || p.index_elems <= 0) return false;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned long long* s_kept = reinterpret_cast<unsigned long long*>(smem_raw);  // scratch before set-up
  if (threadIdx.x == 0) *s_kept = 0ull;
  __syncthreads();
  const long long n = (long long)p.hq * p.seq.total_blocks;
  unsigned long long part = 0ull;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) part += (unsigned)max(__ldg(p.counts + i), 0);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(kFull, part, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(s_kept, part);
  __syncthreads();
  const bool rows = 5ull * *s_kept < 2ull * (unsigned long long)p.index_elems;
  __syncthreads();  // the scratch word is part of the set-up area of either schedule
  return rows;
}

// The paired schedule (every instance); the plain bf16 B = 128 instance returns at once when the row
// schedule is chosen, and attn_rows_kernel, launched right after it, runs the lists instead (two
// kernels, so that each schedule keeps its own code and register allocation).
template <int BK, bool kCache, bool kFp8>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  if constexpr (BK == 128 && !kCache && !kFp8)
    if (rows_chosen(p)) return;
  attn_pairs<BK, kCache, kFp8>(p);
}

__global__ void __launch_bounds__(kThreads, 1) attn_rows_kernel(const __grid_constant__ AttnParams p) {
  if (!rows_chosen(p)) return;
  attn_rows(p);
}

template <int BK, bool kCache, bool kFp8>
static cudaError_t launch_attn_t(const AttnParams& p, int grid, cudaStream_t st) {
  static unsigned long long attr_done[kMaxCachedDevices] = {};
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(attn_kernel<BK, kCache, kFp8>), Cfg<BK, kFp8>::kSmemMax,
                               attr_done);
  if (e != cudaSuccess) return e;
  attn_kernel<BK, kCache, kFp8><<<grid, kThreads, Cfg<BK, kFp8>::smem_bytes(p.seq.num_seqs), st>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if constexpr (BK == 128 && !kCache && !kFp8) {
    if (!p.dense && p.units != 1) {  // the row schedule's kernel (returns at once unless chosen)
      static_assert(rows::smem_bytes(kMaxSeqs) <= 227 * 1024, "shared memory per CTA");
      static unsigned long long attr_rows[kMaxCachedDevices] = {};
      if ((e = set_max_smem(reinterpret_cast<const void*>(attn_rows_kernel), rows::smem_bytes(kMaxSeqs), attr_rows)) !=
          cudaSuccess)
        return e;
      attn_rows_kernel<<<grid, kThreads, rows::smem_bytes(p.seq.num_seqs), st>>>(p);
      e = cudaGetLastError();
    }
  }
  return e;
}

cudaError_t launch_attn(const AttnParams& p, int grid, cudaStream_t st) {
  const bool cache = p.seq.prefix_lens != nullptr || p.seq.block_table != nullptr;
  if (p.fp8) {  // e4m3 Q / K: plain prefill only
    if (cache) return cudaErrorNotSupported;
    return p.seq.block == 128 ? launch_attn_t<128, false, true>(p, grid, st) : launch_attn_t<64, false, true>(p, grid, st);
  }
  if (p.seq.block == 128)
    return cache ? launch_attn_t<128, true, false>(p, grid, st) : launch_attn_t<128, false, false>(p, grid, st);
  return cache ? launch_attn_t<64, true, false>(p, grid, st) : launch_attn_t<64, false, false>(p, grid, st);
}

}  // namespace fp
