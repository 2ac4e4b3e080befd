// Paged decode attention for sm_100a.
//
// What is computed is defined by "Under the Hood: The PagedAttention CUDA
// Kernel" ("PagedAttention and KV Cache Management"): the kernel takes the
// block table as an argument, looks up each logical block's physical block and
// gathers K and V from there, keeping intermediate softmax reductions and
// writing the context vector. The design below is this library's own.
//
// Work decomposition. One work item is one (sequence s, kv head h, logical
// block b) triple; items are ordered s-major, then h, then b, and a unit
// (s, h) owns max(ceil(L_s / B), 1) consecutive items (an empty sequence keeps
// one item so that its output is written). The W items are cut into equal
// contiguous ranges, one per warp of a grid that fills every SM once.
// Equal bytes do not mean equal time: SMs in some GPCs get less DRAM
// bandwidth than others. So a warp claims the items of its range one by one
// from the front of an atomic range word, and a warp that runs out steals the
// back half of the largest unclaimed remainder (a steal is one CAS on that
// word). Every range, own or stolen, is a contiguous sub-range of items; a
// warp writes the output of each unit that lies wholly inside a sub-range it
// processed, and a unit cut by sub-range boundaries leaves fp32 partials
// (m, l, unnormalised O) per piece, which decode_merge_kernel combines.
// Range words and the steal-slot pool start at zero and the merge kernel
// zeroes them again after use; steal records carry a 32-bit call tag.
//
// Per warp: a private ring of NS shared-memory stages. Lane 0 issues the TMA
// tensor loads of one item (the K tile and the V tile of one (block, head):
// B x D elements each) into a stage and arms that stage's mbarrier with the
// byte count; the warp waits on the barrier, computes, and refills the same
// stage NS items ahead. The tiles land 128-byte swizzled, so ldmatrix reads
// are bank-conflict free.
//
// Per item, with the g query heads of the kv head as the N = 8 dimension of
// m16n8k16 MMAs (heads past g are zero):
//   S^T[token, head] = K Q^T           A = K tile (ldmatrix), B = Q^T (registers)
//   online softmax per head over tokens (exp2 domain, warp shuffles)
//   O^T[d, head]    += V^T P^T         A = V tile (ldmatrix.trans), B = P^T
// P^T's B fragment is the transpose of S^T's accumulator layout, one
// movmatrix per 8x8 tile. Slots past the context length are masked by
// predicate: their logits become -inf and their V entries 0, so NaN there
// never reaches the result. fp8-e4m3 tiles are widened to f16 in registers
// (exact); q is rounded to f16 for that path (a bf16 row beyond the f16 range
// is first scaled by a power of two, folded back into that head's logit
// scale) and the per-head scales are folded into the logit scale and the
// output.
#pragma once

#include <type_traits>

#include "ptx.cuh"

namespace pkv {

enum CacheKind : int { kCacheF16 = 0, kCacheBF16 = 1, kCacheE4M3 = 2 };

constexpr int kMaxSteals = 6;     // steals from one warp's range per call
constexpr int kMinStealable = 4;  // a remainder worth splitting (items)
constexpr int kStealMax = 8;      // items one steal takes at most
// The merge's CTA 0 keeps each of its threads' ranges of the adaptive
// partition in registers: at most this many per thread (grids of up to
// 128 x kAdaptPer warps).
constexpr int kAdaptPer = 16;
constexpr int kStealTries = 8;
constexpr int kScanBatch = 4;     // range words each lane loads when choosing a victim (a window of 128)
constexpr int kMergeAhead = 8;    // ranges whose steal records the merge reads in its first round
constexpr int kErrBadMerge = 16;  // a merge record out of range (skipped)

struct DecodeParams {
  CUtensorMap tmk;  // K pool viewed as {D, B, Hk, NB}
  CUtensorMap tmv;  // V pool
  const void* q;
  long long q_s, q_h;  // element strides of q [S, Hq, D]
  void* out;
  long long o_s, o_h;
  const int* tables;
  long long t_s;  // row stride of block_tables
  const int* lens;
  const float* k_scale;  // fp8 only
  const float* v_scale;
  float scale_log2;  // softmax scale * log2(e)
  int S, Hk, g, MB, NB;
  int nwt;                    // consumer warps in the grid
  int tag;                    // per-call tag of steal records (never 0)
  int steal;                  // 1: warps that run out of work steal; 0: static split only
  int pool_slots;             // partial slots available to steals
  long long* hdr;             // workspace header: [0] total items W
  int* err;                   // device-check flag (OR of error bits)
  unsigned long long* words;  // [nwt] range word: front | back | steals; 0 between calls
  unsigned* pool;             // steal-slot pool counter; 0 between calls
  int4* steal_info;           // [nwt][kMaxSteals] (start lo, slot base, tag, start hi)
  int4* desc;                 // [nwt][1 + kMaxSteals] last-piece descriptor per sub-range
  long long* rlo;             // [nwt + 1] first item of each static warp range (the last: W)
  // Adaptive partition (adapt = 1, with work stealing): when *part_nwt ==
  // nwt, static range v starts at item floor(W * part[v] / 2^32) (part[0] =
  // 0, range nwt ends at W); part was computed by the previous call's merge
  // from the running weights wgt[gw] and each warp's predicted time for its
  // whole range, rtime[gw] (us: from its start to the end of its own part,
  // scaled by the items assigned over the items it processed itself).
  // Otherwise the ranges are equal.
  int adapt;
  const int* part_nwt;
  const unsigned* part;       // [nwt]
  float* rtime;               // [nwt]
  float* wgt;                 // [nwt]
  int* part_nwt_w;            // the same word, written by the merge
  unsigned* part_w;
  float* part_o;              // [2 nwt + pool_slots][g][D]
  float* part_ml;             // [2 nwt + pool_slots][g][2]
  // Prefix-aware decode (null otherwise): the first skip[s] table entries of
  // sequence s are a shared prefix attended elsewhere; its remaining tokens
  // leave fp32 partials (m, l, unnormalised O) per query head in cas_o /
  // cas_ml instead of an output row when skip[s] > 0.
  const int* skip;            // [S] blocks
  float* cas_o;               // [S * Hq][D]
  float* cas_ml;              // [S * Hq][2]
};

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Warp-uniform bounded wait on an mbarrier phase. Returns false if it did not
// complete within `limit_ns`.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if (it == 0) t0 = global_ns();
    else if ((it & 63) == 0 && global_ns() - t0 > limit_ns) return false;
  }
}

// ---- range words: front [0,24) | back [24,48) | steals [48,52)
// front counts items the owner claimed, back items thieves took from the end.
__device__ __forceinline__ unsigned rw_front(unsigned long long w) { return unsigned(w & 0xffffffu); }
__device__ __forceinline__ unsigned rw_back(unsigned long long w) {
  return unsigned((w >> 24) & 0xffffffu);
}
__device__ __forceinline__ unsigned rw_steals(unsigned long long w) {
  return unsigned((w >> 48) & 0xfu);
}
__device__ __forceinline__ unsigned long long rw_make(unsigned front, unsigned back, unsigned steals) {
  return static_cast<unsigned long long>(front) | (static_cast<unsigned long long>(back) << 24) |
         (static_cast<unsigned long long>(steals) << 48);
}
__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

template <int BS>
__device__ __forceinline__ int items_of(int L) {
  int n = (L + BS - 1) / BS;
  return n > 0 ? n : 1;
}

// Tokens of sequence s this kernel attends (its context length clamped to the
// table row, minus a shared prefix of sk blocks), and sk.
template <int BS>
__device__ __forceinline__ int seq_len(const DecodeParams& p, int s, int max_len, int& sk,
                                       bool report) {
  int len = __ldg(p.lens + s);
  bool bad = len < 0 || len > max_len;
  len = len < 0 ? 0 : (len > max_len ? max_len : len);
  sk = 0;
  if (p.skip) {
    sk = __ldg(p.skip + s);
    if (sk < 0 || sk * BS > len) {
      bad = true;
      sk = sk < 0 ? 0 : len / BS;
    }
  }
  if (bad && report) atomicOr(p.err, kErrBadLen);
  return len - sk * BS;
}

__device__ __forceinline__ long long range_lo(long long w, long long W, int nwt) {
  return (w * W) / nwt;
}

template <int BS, int TOK>
struct Cursor {
  long long k;  // global item index
  int s, h, b;  // sequence, kv head, item within the unit
  int L, n;     // tokens of s attended here, items per unit of s
  int sk;       // table entries of s skipped (shared prefix)

  __device__ __forceinline__ void advance(const DecodeParams& p, int max_len) {
    ++k;
    if (++b == n) {
      b = 0;
      if (++h == p.Hk) {
        h = 0;
        if (++s < p.S) {
          L = seq_len<BS>(p, s, max_len, sk, false);
          n = items_of<TOK>(L);
        }
      }
    }
  }
  __device__ __forceinline__ long long unit_begin() const { return k - b; }
  __device__ __forceinline__ long long unit_end() const { return k - b + n; }
};

template <int CK, bool QBF, int D, int BS, int NC, int NS, int IB>
struct DecodeCfg {
  static constexpr bool kFp8 = (CK == kCacheE4M3);
  static constexpr bool kMmaBF16 = (CK == kCacheBF16);
  static constexpr int EB = kFp8 ? 1 : 2;         // cache element bytes
  static constexpr int EPR = 128 / EB;            // elements per swizzled 128-byte row
  static constexpr int NH = (D * EB) / 128;       // 128-byte column groups per token row
  static constexpr int TILE = BS * D * EB;        // one K (or V) tile of one block
  static constexpr int TOK = IB * BS;             // tokens per work item
  static constexpr int KT = IB * TILE;            // K (or V) tiles of one item
  static constexpr int STAGE = 2 * KT;
  static constexpr int KS = D / 16;               // k-steps of the QK^T product
  static constexpr int MT = D / 16;               // m-tiles of the PV product
  static constexpr int TT = TOK / 16;             // 16-token tiles per item
  static constexpr int NT = NC * 32;
  static constexpr int SMEM = 1024 + NC * NS * STAGE + NC * NS * 8 + (NT + NC + 1) * 8 + 64;
  static_assert((D * EB) % 128 == 0, "head_dim * elem bytes must be a multiple of 128");
  static_assert(BS % 16 == 0, "block_size must be a multiple of 16");
  static_assert(TILE % 1024 == 0, "tiles must keep 1 KiB swizzle alignment");
  static_assert(NS >= 2, "the claim pipeline needs two stages");
};

// Byte offset of 16-byte chunk `bcol / 16` of token row `t` inside a tile
// loaded with 128-byte swizzle as NH column groups of [BS rows x 128 B].
template <int BS>
__device__ __forceinline__ uint32_t swz(int t, int bcol) {
  return static_cast<uint32_t>((bcol >> 7) * (BS * 128) + t * 128 +
                               ((((bcol & 127) >> 4) ^ (t & 7)) << 4));
}

template <int CK, bool QBF, int D, int BS, int NC, int NS, int IB>
__global__ void __launch_bounds__(NC * 32, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecodeCfg<CK, QBF, D, BS, NC, NS, IB>;
  constexpr int TOK = C::TOK;
  constexpr bool FP8 = C::kFp8;
  constexpr bool MBF = C::kMmaBF16;
  constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - smem_addr(smem_raw));
  const uint32_t stages = sbase;
  const uint32_t bars = sbase + NC * NS * C::STAGE;
  long long* scan = reinterpret_cast<long long*>(sgen + NC * NS * C::STAGE + NC * NS * 8);
  long long* wbase = scan + C::NT;
  long long* total = wbase + NC;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int r = lane >> 2;  // MMA group id
  const int c = lane & 3;   // thread in group
  const int max_len = p.MB * BS;

  // The merge kernel may be scheduled now; it waits for this grid to finish.
  pdl_launch_dependents();

  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(bars + (warp * NS + i) * 8, 1);
  }
  if (tid == 0) {
    tma_prefetch_desc(&p.tmk);
    tma_prefetch_desc(&p.tmv);
  }
  fence_mbar_init();
  // This grid may have started before the previous kernel in the stream
  // finished (programmatic dependent launch): nothing above touches global
  // memory; everything below may.
  pdl_wait();

  // The owner's first claim on its range word (NS items, see run_range) goes
  // out now so its round trip overlaps the length scan below.
  const int gw = blockIdx.x * NC + warp;
  const uint64_t t_start = global_ns();
  unsigned long long first_claim = 0;
  if (p.steal && lane == 0) first_claim = atomicAdd(p.words + gw, static_cast<unsigned long long>(NS));

  // ---- total work and each thread's chunk prefix (every CTA, redundantly) ----
  {
    const int s0 = static_cast<int>((static_cast<long long>(tid) * p.S) / C::NT);
    const int s1 = static_cast<int>((static_cast<long long>(tid + 1) * p.S) / C::NT);
    long long sum = 0;
    for (int s = s0; s < s1; ++s) {
      int sk;
      const int len = seq_len<BS>(p, s, max_len, sk, blockIdx.x == 0);
      sum += static_cast<long long>(p.Hk) * items_of<TOK>(len);
    }
    long long v = sum;  // inclusive warp scan, then warp totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    scan[tid] = v;
    __syncthreads();
    if (tid == 0) {
      long long run = 0;
      for (int w = 0; w < NC; ++w) {
        wbase[w] = run;
        run += scan[w * 32 + 31];
      }
      *total = run;
    }
    __syncthreads();
    scan[tid] = v - sum + wbase[warp];  // exclusive prefix of this thread's chunk
    __syncthreads();
  }
  const long long W = *total;
  if (blockIdx.x == 0 && tid == 0) p.hdr[0] = W;

  // first item of static range v (0 <= v <= nwt)
  const bool adapt = p.adapt && p.steal && __ldcg(p.part_nwt) == p.nwt;
  auto rlo_of = [&](int v) -> long long {
    if (!adapt) return range_lo(v, W, p.nwt);
    if (v >= p.nwt) return W;
    return static_cast<long long>(__umul64hi(static_cast<unsigned long long>(W),
                                             static_cast<unsigned long long>(__ldcg(p.part + v)) << 32));
  };
  const long long my_lo = rlo_of(gw);
  const long long my_len = rlo_of(gw + 1) - my_lo;
  if (my_len >= (1ll << 23)) {  // range words hold 24-bit counts
    if (lane == 0) atomicOr(p.err, kErrBadLen);
    return;
  }

  if (lane == 0) {
    p.desc[gw * (1 + kMaxSteals)] = make_int4(-1, 0, 0, 0);
    p.rlo[gw] = my_lo;  // the merge reads the range boundaries instead of dividing
    if (gw == p.nwt - 1) p.rlo[p.nwt] = W;
  }

  // Position of global item x: chunk by binary search, then a warp-wide walk.
  auto locate = [&](long long x, Cursor<BS, TOK>& out) -> bool {
    int a = 0, bnd = C::NT - 1;
    while (a < bnd) {  // largest t with scan[t] <= x
      int m = (a + bnd + 1) >> 1;
      if (scan[m] <= x) a = m;
      else bnd = m - 1;
    }
    const int s_lo = static_cast<int>((static_cast<long long>(a) * p.S) / C::NT);
    const int s_hi = static_cast<int>((static_cast<long long>(a + 1) * p.S) / C::NT);
    long long base = scan[a];
    for (int s0 = s_lo; s0 < s_hi; s0 += 32) {
      const int s = s0 + lane;
      int len = 0, sk = 0;
      long long w = 0;
      if (s < s_hi) {
        len = seq_len<BS>(p, s, max_len, sk, false);
        w = static_cast<long long>(p.Hk) * items_of<TOK>(len);
      }
      long long incl = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, s < s_hi && base + incl > x);
      if (hit) {
        const int j = __ffs(hit) - 1;
        const long long start = __shfl_sync(0xffffffffu, base + incl - w, j);
        const int L = __shfl_sync(0xffffffffu, len, j);
        out.sk = __shfl_sync(0xffffffffu, sk, j);
        const int n = items_of<TOK>(L);
        const long long off = x - start;
        out.k = x;
        out.s = s0 + j;
        out.h = static_cast<int>(off / n);
        out.b = static_cast<int>(off % n);
        out.L = L;
        out.n = n;
        return true;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    return false;
  };

  const uint64_t policy = l2_policy_evict_first();
  const uint32_t my_stages = stages + warp * NS * C::STAGE;
  const uint32_t my_bars = bars + warp * NS * 8;

  // Table-entry window of the producer: lane j holds table[tw_s][tw_b0 + j].
  int tw_s = -1, tw_b0 = 0, tw_val = 0;
  long long it = 0;      // items consumed by this warp (ring position)
  long long issued = 0;  // items issued into the ring

  uint32_t qb[C::KS][2];
  // q words of the next unit, loaded when its first item is issued (NS - 1
  // items before it is consumed) so the load's latency hides under them;
  // one unit at a time (qn_unit = s * Hk + h, or -1 when free).
  uint32_t qn[C::KS][2];
  int qn_unit = -1;
  // The q words this thread holds of unit (s, h): head r = lane / 4 of the
  // group (zero past g); 16-bit q: two element pairs per 16-dim step, fp8
  // path: four consecutive elements per 16-dim step.
  auto load_q_raw = [&](int s, int h, uint32_t (&raw)[C::KS][2]) {
    const bool row_ok = r < p.g;
    const long long qoff = s * p.q_s + (static_cast<long long>(h) * p.g + r) * p.q_h;
    if constexpr (!FP8) {
      const uint32_t* qp = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.q) + qoff);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        raw[ks][0] = row_ok ? __ldg(qp + (ks * 16 + 2 * c) / 2) : 0u;
        raw[ks][1] = row_ok ? __ldg(qp + (ks * 16 + 8 + 2 * c) / 2) : 0u;
      }
    } else {
      const uint2* qp = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.q) + qoff);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        const uint2 v = row_ok ? __ldg(qp + (ks * 16 + 4 * c) / 4) : make_uint2(0u, 0u);
        raw[ks][0] = v.x;
        raw[ks][1] = v.y;
      }
    }
  };
  float acc[C::MT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float sl0 = p.scale_log2, sl1 = p.scale_log2;  // logit scales of head columns 2c and 2c + 1
  const bool h0_ok = (2 * c) < p.g;
  const bool h1_ok = (2 * c + 1) < p.g;

  // Process the sub-range [a, hi) of warp `owner`'s static range as its
  // `sub`-th sub-range (0 = the owner's own front part, j + 1 = steal j).
  // In claim mode the items are claimed one by one from the range word, and
  // hi drops to where thieves took over. Partials go to slots slot_base (+1).
  auto run_range = [&](long long a, long long hi, bool claim, int owner, int sub,
                       long long slot_base) -> bool {
    Cursor<BS, TOK> cur;
    if (!locate(a, cur)) {
      if (lane == 0) atomicOr(p.err, kErrBadLen);
      return false;
    }
    Cursor<BS, TOK> pc = cur;
    const long long lo = a;

    unsigned long long* wp = p.words + owner;
    const unsigned own_len = static_cast<unsigned>(hi - a);
    bool claiming = claim;
    // Claims: lane 0's `pend` is the range word as the latest claim found
    // it; that claim covers pend_n items, pend_off of them issued so far. The
    // first claim (NS items) was made at the kernel's start, later ones take
    // one item each.
    unsigned long long pend = first_claim;
    int pend_off = 0, pend_n = NS;

    auto issue = [&](int stage) {
      if ((pc.b == 0 || pc.k == lo) && qn_unit < 0) {  // the first item of a unit: its q
        load_q_raw(pc.s, pc.h, qn);
        qn_unit = pc.s * p.Hk + pc.h;
      }
      const uint32_t bar = my_bars + stage * 8;
      if (pc.L == 0) {
        if (lane == 0) mbar_arrive(bar);
        return;
      }
      // blocks b0 .. b0 + nload - 1 of the sequence: the item's blocks that hold tokens
      const int nb = (pc.L + BS - 1) / BS;
      const int b0 = pc.b * IB;
      const int nload = min(IB, nb - b0);
      if (pc.s != tw_s || b0 < tw_b0 || b0 + nload > tw_b0 + 32) {
        tw_s = pc.s;
        tw_b0 = b0;
        tw_val = (tw_b0 + lane < nb) ? __ldg(p.tables + pc.s * p.t_s + pc.sk + tw_b0 + lane) : 0;
      }
      int phys[IB];
#pragma unroll
      for (int ib = 0; ib < IB; ++ib) {
        phys[ib] = __shfl_sync(0xffffffffu, tw_val, (b0 - tw_b0 + ib) & 31);
        if (ib < nload && (phys[ib] < 0 || phys[ib] >= p.NB)) {
          if (lane == 0) atomicOr(p.err, kErrBadBlock);
          phys[ib] = 0;
        }
      }
      if (lane == 0) {
        const uint32_t dk = my_stages + stage * C::STAGE;
        const uint32_t dv = dk + C::KT;
        mbar_arrive_expect_tx(bar, nload * 2 * C::TILE);
#pragma unroll
        for (int ib = 0; ib < IB; ++ib) {
          if (ib < nload) {
#pragma unroll
            for (int hh = 0; hh < C::NH; ++hh)
              tma_load_4d(dk + ib * C::TILE + hh * BS * 128, &p.tmk, bar, hh * C::EPR, 0, pc.h,
                          phys[ib], policy);
#pragma unroll
            for (int hh = 0; hh < C::NH; ++hh)
              tma_load_4d(dv + ib * C::TILE + hh * BS * 128, &p.tmv, bar, hh * C::EPR, 0, pc.h,
                          phys[ib], policy);
          }
        }
      }
    };
    // Issue the item at pc into the next ring stage if it is ours; false when
    // the sub-range has ended.
    auto try_issue = [&]() -> bool {
      if (pc.k >= hi) return false;
      if (claiming) {
        const unsigned long long w =
            __shfl_sync(0xffffffffu, pend, 0) + static_cast<unsigned long long>(pend_off);
        if (rw_front(w) + rw_back(w) >= own_len) {
          claiming = false;
          hi = pc.k;  // everything from here on belongs to thieves
          return false;
        }
      }
      issue(static_cast<int>(issued % NS));
      pc.advance(p, max_len);
      ++issued;
      if (claiming && ++pend_off == pend_n) {  // claim the following item
        pend_off = 0;
        pend_n = 1;
        if (lane == 0) pend = atomicAdd(wp, 1ull);
      }
      return true;
    };

    if (lane == 0) p.desc[owner * (1 + kMaxSteals) + sub] = make_int4(-1, 0, 0, 0);
    for (int i = 0; i < NS; ++i)
      if (!try_issue()) break;

    auto begin_unit = [&]() {
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      float sl = p.scale_log2;
      if constexpr (FP8) sl *= __ldg(p.k_scale + cur.h);
      sl0 = sl1 = sl;
      uint32_t raw[C::KS][2];
      if (qn_unit == cur.s * p.Hk + cur.h) {  // prefetched at issue
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
          raw[ks][0] = qn[ks][0];
          raw[ks][1] = qn[ks][1];
        }
        qn_unit = -1;
      } else {
        load_q_raw(cur.s, cur.h, raw);
      }
      if constexpr (!FP8) {
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
          qb[ks][0] = raw[ks][0];
          qb[ks][1] = raw[ks][1];
        }
      } else {
        // k-slot order of the widened fp8 tile: slots 2c, 2c+1 <- dims 4c, 4c+1
        // and slots 2c+8, 2c+9 <- dims 4c+2, 4c+3 of each 16-dim step.
        float f[C::KS][4];
        float amax = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
          uint2 v = make_uint2(raw[ks][0], raw[ks][1]);
          if constexpr (QBF) {
            f[ks][0] = __uint_as_float(v.x << 16);
            f[ks][1] = __uint_as_float(v.x & 0xffff0000u);
            f[ks][2] = __uint_as_float(v.y << 16);
            f[ks][3] = __uint_as_float(v.y & 0xffff0000u);
          } else {
            __half2 a2 = *reinterpret_cast<__half2*>(&v.x);
            __half2 b2 = *reinterpret_cast<__half2*>(&v.y);
            f[ks][0] = __low2float(a2);
            f[ks][1] = __high2float(a2);
            f[ks][2] = __low2float(b2);
            f[ks][3] = __high2float(b2);
          }
          if constexpr (QBF)
            amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f[ks][0]), fabsf(f[ks][1])),
                                     fmaxf(fabsf(f[ks][2]), fabsf(f[ks][3]))));
        }
        // q rounded to f16. A bf16 row may exceed the f16 range (2^16 and
        // up): it is scaled by a power of two 2^-e (exact) and its logit
        // scale by 2^e. Rows below 2^16 keep e = 0. The row of head r is held
        // by lanes 4r .. 4r + 3.
        float qs = 1.f;
        if constexpr (QBF) {
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
          const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
          const int e = ex >= 16 ? ex - 15 : 0;
          qs = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
          const int e0 = __shfl_sync(0xffffffffu, e, 8 * c), e1 = __shfl_sync(0xffffffffu, e, 8 * c + 4);
          sl0 = sl * __uint_as_float(static_cast<uint32_t>(127 + e0) << 23);
          sl1 = sl * __uint_as_float(static_cast<uint32_t>(127 + e1) << 23);
        }
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
          qb[ks][0] = pack2<false>(f[ks][0] * qs, f[ks][1] * qs);
          qb[ks][1] = pack2<false>(f[ks][2] * qs, f[ks][3] * qs);
        }
      }
    };

    auto finish_unit = [&]() {
      // full row sums per head: reduce the thread partials over the 8 row groups
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
      }
      float vs = 1.f;
      if constexpr (FP8) vs = __ldg(p.v_scale + cur.h);
      const long long ub = cur.unit_begin(), ue = cur.unit_end();
      const int hq0 = cur.h * p.g + 2 * c;
      if (ub >= lo && ue <= hi && cur.sk > 0) {
        // whole unit of a sequence with a shared prefix: its partial goes to
        // the prefix-aware merge
        const long long row = static_cast<long long>(cur.s) * p.g * p.Hk + hq0;
        float* po = p.cas_o + row * D;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
          const int db = FP8 ? da + 1 : da + 8;
          if (h0_ok) {
            po[da] = acc[mt][0] * vs;
            po[db] = acc[mt][2] * vs;
          }
          if (h1_ok) {
            po[D + da] = acc[mt][1] * vs;
            po[D + db] = acc[mt][3] * vs;
          }
        }
        if (r == 0) {
          float* pm = p.cas_ml + row * 2;
          if (h0_ok) {
            pm[0] = m0;
            pm[1] = l0;
          }
          if (h1_ok) {
            pm[2] = m1;
            pm[3] = l1;
          }
        }
      } else if (ub >= lo && ue <= hi) {  // whole unit in this sub-range: final output
        const float i0 = l0 > 0.f ? vs / l0 : 0.f;
        const float i1 = l1 > 0.f ? vs / l1 : 0.f;
        uint16_t* o = static_cast<uint16_t*>(p.out) + cur.s * p.o_s;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
          const int db = FP8 ? da + 1 : da + 8;
          if (h0_ok) {
            uint16_t* oh = o + hq0 * p.o_h;
            const float x = acc[mt][0] * i0, y = acc[mt][2] * i0;
            if constexpr (QBF) {
              oh[da] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
              oh[db] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
            } else {
              oh[da] = __half_as_ushort(__float2half_rn(x));
              oh[db] = __half_as_ushort(__float2half_rn(y));
            }
          }
          if (h1_ok) {
            uint16_t* oh = o + (hq0 + 1) * p.o_h;
            const float x = acc[mt][1] * i1, y = acc[mt][3] * i1;
            if constexpr (QBF) {
              oh[da] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
              oh[db] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
            } else {
              oh[da] = __half_as_ushort(__float2half_rn(x));
              oh[db] = __half_as_ushort(__float2half_rn(y));
            }
          }
        }
      } else {  // piece of a cut unit: fp32 partials for the merge kernel
        const int slot = ub < lo ? 0 : 1;
        const long long base = (slot_base + slot) * p.g;
        float* po = p.part_o + base * D;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
          const int db = FP8 ? da + 1 : da + 8;
          if (h0_ok) {
            po[(2 * c) * D + da] = acc[mt][0] * vs;
            po[(2 * c) * D + db] = acc[mt][2] * vs;
          }
          if (h1_ok) {
            po[(2 * c + 1) * D + da] = acc[mt][1] * vs;
            po[(2 * c + 1) * D + db] = acc[mt][3] * vs;
          }
        }
        if (r == 0) {
          float* pm = p.part_ml + base * 2;
          if (h0_ok) {
            pm[(2 * c) * 2 + 0] = m0;
            pm[(2 * c) * 2 + 1] = l0;
          }
          if (h1_ok) {
            pm[(2 * c + 1) * 2 + 0] = m1;
            pm[(2 * c + 1) * 2 + 1] = l1;
          }
        }
        if (slot == 1 && lane == 0)
          p.desc[owner * (1 + kMaxSteals) + sub] =
              make_int4(cur.s, cur.h, static_cast<int>(ue & 0xffffffffll),
                        static_cast<int>(ue >> 32));
      }
    };

    // ---- main loop over the sub-range ----
    while (cur.k < hi) {
      if (cur.b == 0 || cur.k == lo) begin_unit();
      const int stage = static_cast<int>(it % NS);
      const uint32_t parity = static_cast<uint32_t>((it / NS) & 1);
      if (!warp_wait(my_bars + stage * 8, parity, kWaitNs)) {
        if (lane == 0) atomicOr(p.err, kErrWaitTimeout);
        for (long long j = it + 1; j < issued; ++j)  // let copies in flight land
          warp_wait(my_bars + static_cast<int>(j % NS) * 8, static_cast<uint32_t>((j / NS) & 1),
                    100000000ull);
        return false;
      }


      bool refilled = false;
      if (cur.L > 0) {
        const uint32_t tk = my_stages + stage * C::STAGE;
        const uint32_t tv = tk + C::KT;
        const int nvalid = min(TOK, cur.L - cur.b * TOK);
        // 16-token blocks: the V fragments go to registers right after QK^T
        // (the MMAs consume the K fragments, the context mask consumes the V
        // fragments), so the stage is refilled before the softmax and PV and
        // stays in flight for longer.
        constexpr bool kEarly = (C::TT == 1);
        constexpr int VF = FP8 ? C::MT / 2 : C::MT;  // ldmatrix.x4 of one V tile
        uint32_t vf[kEarly ? VF : 1][FP8 ? 8 : 4];

        // S^T = K Q^T
        float sacc[C::TT][4];
#pragma unroll
        for (int tt = 0; tt < C::TT; ++tt) {
          sacc[tt][0] = sacc[tt][1] = sacc[tt][2] = sacc[tt][3] = 0.f;
          // 16-token tile tt lies inside block (tt * 16) / BS of the item
          const uint32_t kt = tk + ((tt * 16) / BS) * C::TILE;
          const int trow = (tt * 16) % BS + (lane & 7) + ((lane >> 3) & 1) * 8;
          if constexpr (!FP8) {
#pragma unroll
            for (int ks = 0; ks < C::KS; ++ks) {
              uint32_t a0, a1, a2, a3;
              ldsm_x4(kt + swz<BS>(trow, ks * 32 + (lane >> 4) * 16), a0, a1, a2, a3);
              mma16816<MBF>(sacc[tt], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
            }
          } else {
#pragma unroll
            for (int kp = 0; kp < C::KS / 2; ++kp) {
              uint32_t x0, x1, x2, x3;
              ldsm_x4(kt + swz<BS>(trow, kp * 32 + (lane >> 4) * 16), x0, x1, x2, x3);
              uint32_t a0, a2, a1, a3, b0, b2, b1, b3;
              e4m3x4_to_f16x2x2(x0, a0, a2);
              e4m3x4_to_f16x2x2(x1, a1, a3);
              e4m3x4_to_f16x2x2(x2, b0, b2);
              e4m3x4_to_f16x2x2(x3, b1, b3);
              mma16816<false>(sacc[tt], a0, a1, a2, a3, qb[2 * kp][0], qb[2 * kp][1]);
              mma16816<false>(sacc[tt], b0, b1, b2, b3, qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
            }
          }
        }

        // V fragments of tile tt (rows tt*16..), tokens past the context
        // zeroed (a NaN there times p = 0 would still be NaN); only an item
        // with such tokens (mask_tag true) pays for the masking. Non-fp8:
        // four A registers per m-tile; fp8: eight (two m-tiles), widened to f16.
        const bool full = nvalid == TOK;  // warp-uniform
        auto load_v = [&](int tt, int i, uint32_t* f, auto mask_tag) {
          constexpr bool kMask = decltype(mask_tag)::value;
          const int tb = tt * 16 + 2 * c;  // tokens of this thread's A halves
          const uint32_t keep01 = !kMask ? 0xffffffffu :
              (tb < nvalid ? 0x0000ffffu : 0u) | (tb + 1 < nvalid ? 0xffff0000u : 0u);
          const uint32_t keep23 = !kMask ? 0xffffffffu :
              (tb + 8 < nvalid ? 0x0000ffffu : 0u) | (tb + 9 < nvalid ? 0xffff0000u : 0u);
          if constexpr (!FP8) {
            const int vrow = (tt * 16) % BS + (lane & 7) + ((lane >> 4) & 1) * 8;
            ldsm_x4_t(tv + ((tt * 16) / BS) * C::TILE + swz<BS>(vrow, i * 32 + ((lane >> 3) & 1) * 16),
                      f[0], f[1], f[2], f[3]);
            if constexpr (kMask) {
              f[0] &= keep01;
              f[1] &= keep01;
              f[2] &= keep23;
              f[3] &= keep23;
            }
          } else {
            const int vrow = (tt * 16) % BS + (lane & 7) + ((lane >> 3) & 1) * 8;
            uint32_t x0, x1, x2, x3;
            ldsm_x4_t(tv + ((tt * 16) / BS) * C::TILE + swz<BS>(vrow, i * 32 + (lane >> 4) * 16), x0,
                      x1, x2, x3);
            // bytes (d, t), (d + 1, t), (d, t + 1), (d + 1, t + 1) -> token
            // pairs (d, t | t + 1) and (d + 1, t | t + 1)
            e4m3x4_to_f16x2x2(prmt(x0, 0, 0x3120), f[0], f[1]);
            e4m3x4_to_f16x2x2(prmt(x1, 0, 0x3120), f[2], f[3]);
            e4m3x4_to_f16x2x2(prmt(x2, 0, 0x3120), f[4], f[5]);
            e4m3x4_to_f16x2x2(prmt(x3, 0, 0x3120), f[6], f[7]);
            if constexpr (kMask) {
              f[0] &= keep01;
              f[1] &= keep01;
              f[2] &= keep23;
              f[3] &= keep23;
              f[4] &= keep01;
              f[5] &= keep01;
              f[6] &= keep23;
              f[7] &= keep23;
            }
          }
        };
        if constexpr (kEarly) {
          if (full) {
#pragma unroll
            for (int i = 0; i < VF; ++i) load_v(0, i, vf[i], std::false_type{});
          } else {
#pragma unroll
            for (int i = 0; i < VF; ++i) load_v(0, i, vf[i], std::true_type{});
          }
          __syncwarp();
          try_issue();  // every read of this stage has completed: refill it
          refilled = true;
        }

        // online softmax over this block's tokens, per head column. The fp8
        // kernel is bound by issue (the widening), so it takes the shorter
        // form: one-instruction exponentials, the context mask only on an
        // item that holds tokens past L, and a lazily moved exponent base.
        // The 16-bit kernels wait on HBM; the shorter form measured slower
        // there (llama3_8b 113.4 -> 115.8 us per step), so they keep the
        // plain one.
        float mx0 = -INFINITY, mx1 = -INFINITY;
        if constexpr (FP8) {
#pragma unroll
          const uint64_t sl2 = f2_pack(sl0, sl1);  // (columns 2c, 2c + 1) pairs: packed f32x2
          for (int tt = 0; tt < C::TT; ++tt) {
            if (full) {
              f2_unpack(f2_mul(f2_pack(sacc[tt][0], sacc[tt][1]), sl2), sacc[tt][0], sacc[tt][1]);
              f2_unpack(f2_mul(f2_pack(sacc[tt][2], sacc[tt][3]), sl2), sacc[tt][2], sacc[tt][3]);
            } else {
              const int t0 = tt * 16 + r, t1 = t0 + 8;
              sacc[tt][0] = t0 < nvalid ? sacc[tt][0] * sl0 : -INFINITY;
              sacc[tt][1] = t0 < nvalid ? sacc[tt][1] * sl1 : -INFINITY;
              sacc[tt][2] = t1 < nvalid ? sacc[tt][2] * sl0 : -INFINITY;
              sacc[tt][3] = t1 < nvalid ? sacc[tt][3] * sl1 : -INFINITY;
            }
            mx0 = fmaxf(mx0, fmaxf(sacc[tt][0], sacc[tt][2]));
            mx1 = fmaxf(mx1, fmaxf(sacc[tt][1], sacc[tt][3]));
          }
          // The exponent base m moves only when a score passes it by more than
          // 8: until then P = 2^(s - m) stays at or below 2^8 (rounded to 16
          // bits with the same relative error, summed in fp32) and neither the
          // column maxima across the warp nor a rescale of O is needed. When
          // it moves it becomes the column's running maximum. (m, l, O) are
          // consistent for any base, which is all the merges use.
          if (__any_sync(0xffffffffu, mx0 > m0 + 8.f || mx1 > m1 + 8.f)) {
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
              mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
              mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
            }
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: nvalid >= 1
            const float al0 = ex2_fast(m0 - mn0), al1 = ex2_fast(m1 - mn1);
            l0 *= al0;
            l1 *= al1;
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) {
              acc[mt][0] *= al0;
              acc[mt][1] *= al1;
              acc[mt][2] *= al0;
              acc[mt][3] *= al1;
            }
            m0 = mn0;
            m1 = mn1;
          }
        } else {
#pragma unroll
          for (int tt = 0; tt < C::TT; ++tt) {
            const int t0 = tt * 16 + r, t1 = t0 + 8;
            sacc[tt][0] = t0 < nvalid ? sacc[tt][0] * sl0 : -INFINITY;
            sacc[tt][1] = t0 < nvalid ? sacc[tt][1] * sl1 : -INFINITY;
            sacc[tt][2] = t1 < nvalid ? sacc[tt][2] * sl0 : -INFINITY;
            sacc[tt][3] = t1 < nvalid ? sacc[tt][3] * sl1 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(sacc[tt][0], sacc[tt][2]));
            mx1 = fmaxf(mx1, fmaxf(sacc[tt][1], sacc[tt][3]));
          }
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: nvalid >= 1
          if (__any_sync(0xffffffffu, mn0 != m0 || mn1 != m1)) {   // a running max moved
            const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
            l0 *= al0;
            l1 *= al1;
#pragma unroll
            for (int mt = 0; mt < C::MT; ++mt) {
              acc[mt][0] *= al0;
              acc[mt][1] *= al1;
              acc[mt][2] *= al0;
              acc[mt][3] *= al1;
            }
            m0 = mn0;
            m1 = mn1;
          }
        }
        uint32_t pb[C::TT][2];
#pragma unroll
        for (int tt = 0; tt < C::TT; ++tt) {
          float p0, p1, p2, p3;
          if constexpr (FP8) {  // exponent arguments and row sums as packed pairs
            const uint64_t nm2 = f2_pack(-m0, -m1);
            float a0, a1, a2, a3;
            f2_unpack(f2_add(f2_pack(sacc[tt][0], sacc[tt][1]), nm2), a0, a1);
            f2_unpack(f2_add(f2_pack(sacc[tt][2], sacc[tt][3]), nm2), a2, a3);
            p0 = ex2_fast(a0);
            p1 = ex2_fast(a1);
            p2 = ex2_fast(a2);
            p3 = ex2_fast(a3);
            f2_unpack(f2_add(f2_pack(l0, l1), f2_add(f2_pack(p0, p1), f2_pack(p2, p3))), l0, l1);
          } else {
            p0 = exp2f(sacc[tt][0] - m0);
            p1 = exp2f(sacc[tt][1] - m1);
            p2 = exp2f(sacc[tt][2] - m0);
            p3 = exp2f(sacc[tt][3] - m1);
            l0 += p0 + p2;
            l1 += p1 + p3;
          }
          pb[tt][0] = movmatrix_t(pack2<MBF>(p0, p1));
          pb[tt][1] = movmatrix_t(pack2<MBF>(p2, p3));
        }

        // O^T += V^T P^T
        auto pv = [&](auto mask_tag) {
#pragma unroll
          for (int tt = 0; tt < C::TT; ++tt) {
#pragma unroll
            for (int i = 0; i < VF; ++i) {
              uint32_t fl[FP8 ? 8 : 4];
              const uint32_t* f = fl;
              if constexpr (kEarly) f = vf[i];
              else load_v(tt, i, fl, mask_tag);
              if constexpr (!FP8) {
                mma16816<MBF>(acc[i], f[0], f[1], f[2], f[3], pb[tt][0], pb[tt][1]);
              } else {
                mma16816<false>(acc[2 * i], f[0], f[1], f[2], f[3], pb[tt][0], pb[tt][1]);
                mma16816<false>(acc[2 * i + 1], f[4], f[5], f[6], f[7], pb[tt][0], pb[tt][1]);
              }
            }
          }
        };
        if (kEarly || full) pv(std::false_type{});
        else pv(std::true_type{});
      }

      if (!refilled) {
        __syncwarp();
        try_issue();  // refill the freed stage NS items ahead
      }
      if (cur.b == cur.n - 1 || cur.k == hi - 1) finish_unit();
      cur.advance(p, max_len);
      ++it;
    }
    return true;
  };

  // ---- own range, then steal until no remainder is worth splitting ----
  if (my_len > 0 && !run_range(my_lo, my_lo + my_len, p.steal != 0, gw, 0, 2ll * gw)) return;
  if (!p.steal) return;  // static split: every unit is cut at the same places in every call
  if (p.adapt && lane == 0) {  // the predicted time of this warp's whole range, for the next call's partition
    const float dt = static_cast<float>(global_ns() - t_start) * 1e-3f;
    p.rtime[gw] = (it > 0 && my_len > 0) ? dt * static_cast<float>(my_len) / static_cast<float>(it) : 0.f;
  }

  // Two partial slots from the pool per steal, reserved only once a victim
  // is in sight and kept across failed attempts (a reservation made for
  // nothing would use up the pool: every warp ends with a failed search).
  unsigned slot0 = 0;
  bool have_slots = false;
  for (int attempt = 0; attempt < 4 * kStealTries; ++attempt) {
    // find the victim with the largest unclaimed remainder, steal its back half
    int stolen = 0;
    bool pool_empty = false;
    long long sa = 0, sb = 0;
    int victim = -1, sj = 0;
    for (int tries = 0; tries < kStealTries && !stolen; ++tries) {
      const int win0 = static_cast<int>(
          ((static_cast<unsigned>(gw) * 2654435761u) >> 7) +
          static_cast<unsigned>((attempt * kStealTries + tries) * 32 * kScanBatch)) % p.nwt;
      long long best = 0;
      int bv = -1;
      unsigned long long bw = 0;
      // A window of 32 x kScanBatch range words, from an offset that differs
      // per thief and per try: every load is issued before the first is used
      // (one round trip), and a window without a candidate ends the search,
      // so a warp with nothing to steal leaves after one round trip.
      {
        unsigned long long wb[kScanBatch];
        long long vl[kScanBatch];  // the sampled ranges' lengths
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
          const int off = lane + 32 * j;
          const int v = (win0 + off) % p.nwt;
          wb[j] = off < p.nwt ? ld_relaxed(p.words + v) : 0ull;
          vl[j] = rlo_of(v + 1) - rlo_of(v);
        }
#pragma unroll
        for (int j = 0; j < kScanBatch; ++j) {
          const unsigned long long w = wb[j];
          const int off = lane + 32 * j;
          const int v = (win0 + off) % p.nwt;
          long long rem = (off >= p.nwt || rw_steals(w) >= kMaxSteals)
                              ? 0
                              : vl[j] - static_cast<long long>(rw_front(w)) - rw_back(w);
          // Thieves that finish together would all pick the same largest
          // remainder and collide on one word: each scores a victim at its
          // remainder plus up to a quarter of it, by a hash of (thief,
          // victim), so they spread over the victims near the largest.
          if (rem >= kMinStealable) {
            const unsigned hsh = (static_cast<unsigned>(v) * 2654435761u) ^
                                 (static_cast<unsigned>(gw + 1) * 2246822519u);
            rem = rem * 4 + ((rem * static_cast<long long>((hsh >> 24) & 0xffu)) >> 8);
          } else {
            rem = 0;
          }
          if (rem > best) {
            best = rem;
            bv = v;
            bw = w;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const long long ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const unsigned long long ow = __shfl_xor_sync(0xffffffffu, bw, o);
        if (ob > best || (ob == best && ov > bv)) {
          best = ob;
          bv = ov;
          bw = ow;
        }
      }
      if (best < 4 * kMinStealable) break;  // (scores are 4x the remainder or more)
      if (!have_slots) {
        if (lane == 0) slot0 = atomicAdd(p.pool, 2u);
        slot0 = __shfl_sync(0xffffffffu, slot0, 0);
        if (slot0 + 2 > static_cast<unsigned>(p.pool_slots)) {
          pool_empty = true;
          break;
        }
        have_slots = true;
      }
      if (lane == 0) {
        // The owner claims an item every microsecond or so, so the word read
        // by the scan is usually stale by now: a failed CAS returns the
        // current word, which the next attempt takes as its expectation.
        const long long vlo = rlo_of(bv);
        const long long vlen = rlo_of(bv + 1) - vlo;
        unsigned long long cur = bw;
        for (int c = 0; c < kStealTries; ++c) {
          const unsigned f = rw_front(cur), b = rw_back(cur), ns = rw_steals(cur);
          const long long rem = vlen - static_cast<long long>(f) - b;
          if (rem < kMinStealable || ns >= kMaxSteals) break;
          // half the remainder, at most kStealMax items: a stolen range is
          // not stolen from again, so a large late steal becomes the tail
          const unsigned take = static_cast<unsigned>(rem / 2 < kStealMax ? rem / 2 : kStealMax);
          const unsigned long long want = rw_make(f, b + take, ns + 1);
          const unsigned long long prev = atomicCAS(p.words + bv, cur, want);
          if (prev == cur) {
            stolen = 1;
            sb = vlo + vlen - b;
            sa = sb - take;
            victim = bv;
            sj = static_cast<int>(ns);
            p.steal_info[bv * kMaxSteals + sj] =
                make_int4(static_cast<int>(sa & 0xffffffffll), 2 * p.nwt + static_cast<int>(slot0),
                          p.tag, static_cast<int>(sa >> 32));
            break;
          }
          cur = prev;
        }
      }
      stolen = __shfl_sync(0xffffffffu, stolen, 0);
    }
    if (!stolen || pool_empty) break;
    have_slots = false;  // this steal's partials use them
    sa = __shfl_sync(0xffffffffu, sa, 0);
    sb = __shfl_sync(0xffffffffu, sb, 0);
    victim = __shfl_sync(0xffffffffu, victim, 0);
    sj = __shfl_sync(0xffffffffu, sj, 0);
    if (!run_range(sa, sb, false, victim, sj + 1, 2ll * p.nwt + static_cast<long long>(slot0)))
      return;
  }
}

// Combine the pieces of every unit cut by sub-range boundaries. One CTA per
// static warp range w0 (all resident at once: few registers, small shared
// memory), organised as a fixed number of memory rounds whose loads are all
// independent: (1) the range's descriptors, steal records and the item count
// together; (2) for each of its sub-ranges whose last piece starts a cut
// unit, the steal records of the following static ranges, one range per
// thread (the next 128, and so on), listing the piece slots of every
// sub-range that starts before the unit's end; (3) the pieces' running
// maxima per head; (4) the rescaled sums. A piece's place in the list comes
// from a block-wide scan (range order, then item order inside a range), so
// the list is the same every time it is built: a unit with more pieces than
// the list holds is folded in several passes over it, and a call without
// steals folds every unit's pieces in one fixed order.
template <bool QBF, int D>
__global__ void __launch_bounds__(128, 8) decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  pdl_wait();  // the decode grid has finished
  pdl_launch_dependents();
  constexpr int NT = 128;
  constexpr int kCap = 1024;  // pieces folded per pass
  constexpr int ND = 1 + kMaxSteals;
  __shared__ int s_slot[kCap];
  __shared__ float s_red[NT * 10];
  __shared__ int s_wsum[NT / 32];
  __shared__ int4 s_desc[ND];
  __shared__ int4 s_rec[kMergeAhead][kMaxSteals];  // steal records of ranges w0 .. w0 + kMergeAhead - 1
  __shared__ long long s_own_start[kMaxSteals];
  __shared__ int s_own_slot[kMaxSteals];
  __shared__ long long s_W;
  __shared__ int s_m_own;
  __shared__ long long s_rlo[NT + 1];  // first items of ranges w0 .. w0 + NT
  constexpr int kSpec = 3;  // pieces loaded speculatively in the first round
  __shared__ float2 s_sp_ml[kSpec][NT];
  __shared__ float4 s_sp_o[kSpec][NT][2];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int w0 = blockIdx.x;
  const int g = p.g;
  const int E = g * D;
  // Thread t owns an 8-element chunk of one head (chunk t % NC8) and the
  // pieces q = t / NC8 (mod PG) of each pass.
  const int NC8 = E / 8;                // chunks of 8 elements (D is a multiple of 8)
  const int PG = NT / NC8;              // piece groups (1 at g = 8, D = 128)
  const int c8 = tid % NC8, pg = tid / NC8;
  const int hi8 = c8 / (D / 8), d8 = (c8 % (D / 8)) * 8;

  // round 1: descriptors, the steal records of this range and the next
  // few (a cut unit rarely reaches further), item count; and, speculatively,
  // the partials of the usual shape of the own part's last cut unit: cut
  // only where the next static ranges begin, its pieces are slots
  // 2 w0 + 1, 2 (w0 + 1), 2 (w0 + 2) (piece group 0 holds them).
  if (pg == 0) {
#pragma unroll
    for (int u = 0; u < kSpec; ++u) {
      const int slot = u == 0 ? 2 * w0 + 1 : 2 * (w0 + u);
      float2 ml = make_float2(-INFINITY, 0.f);
      float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
      if (slot < 2 * p.nwt) {
        const long long base = static_cast<long long>(slot) * g + hi8;
        ml = make_float2(p.part_ml[base * 2], p.part_ml[base * 2 + 1]);
        const float4* op = reinterpret_cast<const float4*>(p.part_o + base * D + d8);
        o0 = op[0];
        o1 = op[1];
      }
      s_sp_ml[u][c8] = ml;
      s_sp_o[u][c8][0] = o0;
      s_sp_o[u][c8][1] = o1;
    }
  }
  if (w0 + tid <= p.nwt) s_rlo[tid] = p.rlo[w0 + tid];
  if (tid == 0 && w0 + NT <= p.nwt) s_rlo[NT] = p.rlo[w0 + NT];
  if (tid < ND) s_desc[tid] = p.desc[w0 * ND + tid];
  else if (tid >= 32 && tid < 32 + kMergeAhead * kMaxSteals) {
    const int j = tid - 32, v = w0 + j / kMaxSteals;
    if (v < p.nwt) s_rec[j / kMaxSteals][j % kMaxSteals] = p.steal_info[v * kMaxSteals + j % kMaxSteals];
  } else if (tid == 32 + kMergeAhead * kMaxSteals) {
    s_W = p.hdr[0];
  } else if (tid == 33 + kMergeAhead * kMaxSteals) {
    p.words[w0] = 0ull;  // leave the claim state zeroed for the next call
    if (w0 == 0) *p.pool = 0u;
  }
  __syncthreads();
  const long long W = s_W;
  // first item of static range v (v <= nwt)
  auto rlo = [&](int v) -> long long { return v - w0 <= NT ? s_rlo[v - w0] : p.rlo[v]; };

  // Steal records j = 0, 1, ... of warp v's range that carry this call's tag,
  // each starting inside v's range with its slots in the pool.
  auto valid_steals = [&](int v, const int4* rec, long long* starts, int* slots) -> int {
    const long long vlo = rlo(v), vhi = rlo(v + 1);
    int m = 0;
    for (int j = 0; j < kMaxSteals; ++j) {
      if (rec[j].z != p.tag) break;
      const long long st = static_cast<long long>(static_cast<unsigned>(rec[j].x)) |
                           (static_cast<long long>(rec[j].w) << 32);
      if (st <= vlo || st >= vhi || rec[j].y < 2 * p.nwt ||
          rec[j].y + 2 > 2 * p.nwt + p.pool_slots) {
        atomicOr(p.err, kErrBadMerge);
        break;
      }
      starts[j] = st;
      slots[j] = rec[j].y;
      m = j + 1;
    }
    return m;
  };

  if (tid == 0) s_m_own = valid_steals(w0, s_rec[0], s_own_start, s_own_slot);
  __syncthreads();
  const int m_own = s_m_own;

  // Piece slots of the sub-ranges of warp range v that start before U1, in
  // item order from its sub-range `from` on (0 = the owner's own part,
  // i >= 1 = steal m - i).
  auto list_range = [&](int v, int from, long long U1, int* out) -> int {
    long long st_v[kMaxSteals];
    int sl_v[kMaxSteals];
    int m;
    if (v == w0) {
      m = m_own;
      for (int j = 0; j < m; ++j) {
        st_v[j] = s_own_start[j];
        sl_v[j] = s_own_slot[j];
      }
    } else if (v < w0 + kMergeAhead) {
      m = valid_steals(v, s_rec[v - w0], st_v, sl_v);
    } else {
      int4 rec[kMaxSteals];
#pragma unroll
      for (int j = 0; j < kMaxSteals; ++j) rec[j] = p.steal_info[v * kMaxSteals + j];
      m = valid_steals(v, rec, st_v, sl_v);
    }
    const long long vlo = rlo(v), vhi = rlo(v + 1);
    int cnt = 0;
    for (int pos = from; pos <= m; ++pos) {
      const long long st = pos == 0 ? vlo : st_v[m - pos];
      const long long en = pos < m ? st_v[m - pos - 1] : vhi;
      if (st >= U1) break;
      if (en > st) out[cnt++] = pos == 0 ? 2 * v : sl_v[m - pos];
    }
    return cnt;
  };

  for (int k = 0; k <= m_own; ++k) {
    const int4 d = s_desc[k];
    if (d.x < 0) continue;
    const int s = d.x, h = d.y;
    const long long U1 = static_cast<long long>(static_cast<unsigned>(d.z)) |
                         (static_cast<long long>(d.w) << 32);
    if (s >= p.S || h < 0 || h >= p.Hk || U1 <= 0 || U1 > W) {
      if (tid == 0) atomicOr(p.err, kErrBadMerge);
      continue;
    }
    // item-order position of this sub-range in w0's list: 0 = owner part,
    // i >= 1 = steal (m - i)
    const int pos0 = (k == 0) ? 0 : m_own - (k - 1);
    const int first = ((k == 0) ? 2 * w0 : s_own_slot[k - 1]) + 1;  // the unit's first piece

    // Each thread loads four of its pieces at a time (m, l and two float4
    // of O each) before folding them with an online max / rescale, then the
    // piece groups are combined.
    float rm = -INFINITY, rl = 0.f, ra[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) ra[x] = 0.f;

    for (int pass = 0;; ++pass) {
      // round 2: list the pieces; this pass keeps positions [wlo, wlo + kCap)
      const int wlo = pass * kCap;
      if (pass == 0 && tid == 0) s_slot[0] = first;
      int run = 1;  // positions taken so far (position 0: the first piece)
      for (int chunk = 0;; ++chunk) {
        const int v = w0 + chunk * NT + tid;
        int sl[ND];
        int cnt = 0;
        if (v < p.nwt && rlo(v) < U1) cnt = list_range(v, v == w0 ? pos0 + 1 : 0, U1, sl);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        if (lane == 31) s_wsum[tid >> 5] = incl;
        __syncthreads();
        int at = run + incl - cnt, tot = 0;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) {
          const int x = s_wsum[w];
          if (w < (tid >> 5)) at += x;
          tot += x;
        }
        for (int i = 0; i < cnt; ++i, ++at)
          if (at >= wlo && at < wlo + kCap) s_slot[at - wlo] = sl[i];
        run += tot;
        __syncthreads();
        const long long next = w0 + static_cast<long long>(chunk + 1) * NT;
        if (next >= p.nwt || rlo(static_cast<int>(next)) >= U1) break;
      }
      const int n = min(run - wlo, kCap);
      // the speculatively loaded pieces are this unit's, in this order
      bool spec = k == 0 && pass == 0 && run <= kSpec;
      for (int u = 1; u < kSpec && spec; ++u)
        spec = u >= run || s_slot[u] == 2 * (w0 + u);
      // rounds 3 and 4: fold this pass's pieces in
      if (spec) {
        if (pg == 0) {
#pragma unroll
          for (int u = 0; u < kSpec; ++u) {
            const float2 ml = s_sp_ml[u][c8];
            if (u >= n || ml.x == -INFINITY) continue;
            const float4 o0 = s_sp_o[u][c8][0], o1 = s_sp_o[u][c8][1];
            const float mn = fmaxf(rm, ml.x);
            const float sa = (rm == -INFINITY) ? 0.f : exp2f(rm - mn), sb = exp2f(ml.x - mn);
            rl = rl * sa + ml.y * sb;
            ra[0] = ra[0] * sa + o0.x * sb;
            ra[1] = ra[1] * sa + o0.y * sb;
            ra[2] = ra[2] * sa + o0.z * sb;
            ra[3] = ra[3] * sa + o0.w * sb;
            ra[4] = ra[4] * sa + o1.x * sb;
            ra[5] = ra[5] * sa + o1.y * sb;
            ra[6] = ra[6] * sa + o1.z * sb;
            ra[7] = ra[7] * sa + o1.w * sb;
            rm = mn;
          }
        }
      } else if (pg < PG) {
        for (int q0 = pg; q0 < n; q0 += 4 * PG) {
          float mv[4], lv[4];
          float4 o0[4], o1[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int q = q0 + u * PG;
            mv[u] = -INFINITY;
            lv[u] = 0.f;
            o0[u] = o1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (q < n) {
              const long long base = static_cast<long long>(s_slot[q]) * g + hi8;
              mv[u] = p.part_ml[base * 2];
              lv[u] = p.part_ml[base * 2 + 1];
              const float4* op = reinterpret_cast<const float4*>(p.part_o + base * D + d8);
              o0[u] = op[0];
              o1[u] = op[1];
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (mv[u] == -INFINITY) continue;
            const float mn = fmaxf(rm, mv[u]);
            const float sa = (rm == -INFINITY) ? 0.f : exp2f(rm - mn), sb = exp2f(mv[u] - mn);
            rl = rl * sa + lv[u] * sb;
            ra[0] = ra[0] * sa + o0[u].x * sb;
            ra[1] = ra[1] * sa + o0[u].y * sb;
            ra[2] = ra[2] * sa + o0[u].z * sb;
            ra[3] = ra[3] * sa + o0[u].w * sb;
            ra[4] = ra[4] * sa + o1[u].x * sb;
            ra[5] = ra[5] * sa + o1[u].y * sb;
            ra[6] = ra[6] * sa + o1[u].z * sb;
            ra[7] = ra[7] * sa + o1[u].w * sb;
            rm = mn;
          }
        }
      }
      __syncthreads();  // the list is rebuilt by the next pass or unit
      if (run <= wlo + kCap) break;
    }
    // combine the piece groups of each chunk
    if (PG > 1) {
      float* red = s_red;  // [NT][10]
      red[tid * 10 + 0] = rm;
      red[tid * 10 + 1] = rl;
#pragma unroll
      for (int x = 0; x < 8; ++x) red[tid * 10 + 2 + x] = ra[x];
      __syncthreads();
      if (pg == 0) {
        for (int gq = 1; gq < PG; ++gq) {
          const float* r2 = red + (gq * NC8 + c8) * 10;
          const float m2 = r2[0];
          if (m2 == -INFINITY) continue;
          const float mn = fmaxf(rm, m2);
          const float sa = (rm == -INFINITY) ? 0.f : exp2f(rm - mn), sb = exp2f(m2 - mn);
          rl = rl * sa + r2[1] * sb;
#pragma unroll
          for (int x = 0; x < 8; ++x) ra[x] = ra[x] * sa + r2[2 + x] * sb;
          rm = mn;
        }
      }
    }
    const bool cascade = p.skip != nullptr && __ldg(p.skip + s) > 0;
    if (pg == 0 && cascade) {  // partial of a sequence with a shared prefix
      const long long row = static_cast<long long>(s) * g * p.Hk + static_cast<long long>(h) * g + hi8;
      float4* po = reinterpret_cast<float4*>(p.cas_o + row * D + d8);
      po[0] = make_float4(ra[0], ra[1], ra[2], ra[3]);
      po[1] = make_float4(ra[4], ra[5], ra[6], ra[7]);
      if (d8 == 0) {
        p.cas_ml[row * 2] = rm;
        p.cas_ml[row * 2 + 1] = rl;
      }
    } else if (pg == 0) {
      const float inv = rl > 0.f ? 1.f / rl : 0.f;
      uint16_t* oh = static_cast<uint16_t*>(p.out) + s * p.o_s +
                     (static_cast<long long>(h) * g + hi8) * p.o_h + d8;
      uint32_t w4[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        if constexpr (QBF) {
          __nv_bfloat162 v2 = __floats2bfloat162_rn(ra[2 * x] * inv, ra[2 * x + 1] * inv);
          w4[x] = *reinterpret_cast<uint32_t*>(&v2);
        } else {
          __half2 v2 = __floats2half2_rn(ra[2 * x] * inv, ra[2 * x + 1] * inv);
          w4[x] = *reinterpret_cast<uint32_t*>(&v2);
        }
      }
      if ((reinterpret_cast<uintptr_t>(oh) & 15) == 0) {
        *reinterpret_cast<uint4*>(oh) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      } else {
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          oh[2 * x] = static_cast<uint16_t>(w4[x] & 0xffffu);
          oh[2 * x + 1] = static_cast<uint16_t>(w4[x] >> 16);
        }
      }
    }
    __syncthreads();  // s_red is reused by the next cut unit
  }

  // CTA 0: the next call's partition from this call's predicted range times
  // T_v. The weight of range v (1 at first) is multiplied by
  // 1 + (mean T / T_v - 1) / 2 (half-way to equal times: one call's times
  // are noisy), the weights are scaled to mean 1 and clamped to [0.5, 2],
  // and range v gets a share of the items proportional to its weight. A
  // range without a time keeps its weight.
  if (blockIdx.x == 0 && p.adapt && p.steal) {
    const int n = p.nwt;
    const int per = (n + NT - 1) / NT;  // at most kAdaptPer: the host enables adapt only then
    if (per > kAdaptPer) return;
    const int va = min(n, tid * per), vb = min(n, va + per);
    const bool have = __ldcg(p.part_nwt) == n;
    double* sd = reinterpret_cast<double*>(s_red);  // [NT / 32] per-warp sums
    // block-wide sum (and the exclusive prefix of this thread) of x
    auto block_scan = [&](double x, double& before, double& all) {
      double incl = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      __syncthreads();
      if (lane == 31) sd[tid >> 5] = incl;
      __syncthreads();
      before = incl - x;
      all = 0.0;
#pragma unroll
      for (int w = 0; w < NT / 32; ++w) {
        if (w < (tid >> 5)) before += sd[w];
        all += sd[w];
      }
    };
    auto valid_time = [](float v) { return v > 0.f && v < 1e9f; };
    // this thread's ranges in registers, every load in flight at once
    float sp[kAdaptPer], w[kAdaptPer];
#pragma unroll
    for (int k = 0; k < kAdaptPer; ++k) {
      const bool in = va + k < vb;
      sp[k] = in ? __ldcg(p.rtime + va + k) : 0.f;
      w[k] = in && have ? __ldcg(p.wgt + va + k) : 1.f;
    }
    double ssum = 0.0, scnt = 0.0, dummy, st, ct;
#pragma unroll
    for (int k = 0; k < kAdaptPer; ++k) {
      if (va + k < vb && valid_time(sp[k])) {
        ssum += sp[k];
        scnt += 1.0;
      }
    }
    block_scan(ssum, dummy, st);
    block_scan(scnt, dummy, ct);
    const float mean = ct > 0.0 ? static_cast<float>(st / ct) : 0.f;
    double wsum = 0.0;
#pragma unroll
    for (int k = 0; k < kAdaptPer; ++k) {
      if (va + k < vb) {
        float wo = w[k];
        if (!(wo >= 0.5f && wo <= 2.f)) wo = 1.f;
        w[k] = (mean > 0.f && valid_time(sp[k])) ? wo * (0.5f + 0.5f * (mean / sp[k])) : wo;
        wsum += w[k];
      }
    }
    double wtot;
    block_scan(wsum, dummy, wtot);
    const float wscale = wtot > 0.0 ? static_cast<float>(n / wtot) : 1.f;
    wsum = 0.0;
#pragma unroll
    for (int k = 0; k < kAdaptPer; ++k) {
      if (va + k < vb) {
        w[k] = fminf(fmaxf(w[k] * wscale, 0.5f), 2.f);
        wsum += w[k];
      }
    }
    double run, total;
    block_scan(wsum, run, total);
#pragma unroll
    for (int k = 0; k < kAdaptPer; ++k) {
      if (va + k < vb) {
        const double f = run / total * 4294967296.0;
        p.part_w[va + k] = f >= 4294967295.0 ? 4294967295u : static_cast<unsigned>(f);
        p.wgt[va + k] = w[k];
        run += w[k];
      }
    }
    if (tid == 0) *p.part_nwt_w = n;
  }
}

}  // namespace pkv
