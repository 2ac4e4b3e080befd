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
// contiguous ranges, one per warp of a grid sized to fill every SM once, so
// every warp streams the same number of KV bytes whatever the length mix.
// A warp writes the output of every unit that lies wholly inside its range;
// a unit cut by a range boundary leaves fp32 partials (m, l, unnormalised O)
// per piece, and decode_merge_kernel combines them.
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
// (exact); q is rounded to f16 for that path and the per-head scales are
// folded into the logit scale and the output.
#pragma once

#include "ptx.cuh"

namespace pkv {

enum CacheKind : int { kCacheF16 = 0, kCacheBF16 = 1, kCacheE4M3 = 2 };

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
  int nwt;            // consumer warps in the grid
  long long* hdr;     // workspace header: [0] total items W
  int* err;           // device-check flag (OR of error bits)
  float* part_o;      // [nwt][2][g][D]
  float* part_ml;     // [nwt][2][g][2]
  int4* desc;         // [nwt] last-segment descriptor (s, h, U1 lo, U1 hi); s < 0: none
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

template <int BS>
__device__ __forceinline__ int items_of(int L) {
  int n = (L + BS - 1) / BS;
  return n > 0 ? n : 1;
}

template <int BS>
struct Cursor {
  long long k;  // global item index
  int s, h, b;  // sequence, kv head, block within the unit
  int L, n;     // context length of s, items per unit of s

  __device__ __forceinline__ void advance(const DecodeParams& p, int max_len) {
    ++k;
    if (++b == n) {
      b = 0;
      if (++h == p.Hk) {
        h = 0;
        if (++s < p.S) {
          int len = __ldg(p.lens + s);
          L = len < 0 ? 0 : (len > max_len ? max_len : len);
          n = items_of<BS>(L);
        }
      }
    }
  }
  __device__ __forceinline__ long long unit_begin() const { return k - b; }
  __device__ __forceinline__ long long unit_end() const { return k - b + n; }
};

template <int CK, bool QBF, int D, int BS, int NC, int NS>
struct DecodeCfg {
  static constexpr bool kFp8 = (CK == kCacheE4M3);
  static constexpr bool kMmaBF16 = (CK == kCacheBF16);
  static constexpr int EB = kFp8 ? 1 : 2;         // cache element bytes
  static constexpr int EPR = 128 / EB;            // elements per swizzled 128-byte row
  static constexpr int NH = (D * EB) / 128;       // 128-byte column groups per token row
  static constexpr int TILE = BS * D * EB;        // one K (or V) tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int KS = D / 16;               // k-steps of the QK^T product
  static constexpr int MT = D / 16;               // m-tiles of the PV product
  static constexpr int TT = BS / 16;              // 16-token tiles per block
  static constexpr int NT = NC * 32;
  static constexpr int SMEM = 1024 + NC * NS * STAGE + NC * NS * 8 + (NT + NC + 1) * 8 + 64;
  static_assert((D * EB) % 128 == 0, "head_dim * elem bytes must be a multiple of 128");
  static_assert(BS % 16 == 0, "block_size must be a multiple of 16");
  static_assert(TILE % 1024 == 0, "tiles must keep 1 KiB swizzle alignment");
};

// Byte offset of 16-byte chunk `bcol / 16` of token row `t` inside a tile
// loaded with 128-byte swizzle as NH column groups of [BS rows x 128 B].
template <int BS>
__device__ __forceinline__ uint32_t swz(int t, int bcol) {
  return static_cast<uint32_t>((bcol >> 7) * (BS * 128) + t * 128 +
                               ((((bcol & 127) >> 4) ^ (t & 7)) << 4));
}

template <int CK, bool QBF, int D, int BS, int NC, int NS>
__global__ void __launch_bounds__(NC * 32) decode_kernel(const __grid_constant__ DecodeParams p) {
  using C = DecodeCfg<CK, QBF, D, BS, NC, NS>;
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

  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(bars + (warp * NS + i) * 8, 1);
  }
  if (tid == 0) {
    tma_prefetch_desc(&p.tmk);
    tma_prefetch_desc(&p.tmv);
  }
  fence_mbar_init();

  // ---- total work and each thread's chunk prefix (every CTA, redundantly) ----
  {
    const int s0 = static_cast<int>((static_cast<long long>(tid) * p.S) / C::NT);
    const int s1 = static_cast<int>((static_cast<long long>(tid + 1) * p.S) / C::NT);
    long long sum = 0;
    for (int s = s0; s < s1; ++s) {
      int len = __ldg(p.lens + s);
      if (len < 0 || len > max_len) {
        if (blockIdx.x == 0) atomicOr(p.err, kErrBadLen);
        len = len < 0 ? 0 : max_len;
      }
      sum += static_cast<long long>(p.Hk) * items_of<BS>(len);
    }
    // inclusive warp scan, then warp totals
    long long v = sum;
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

  const int gw = blockIdx.x * NC + warp;
  const long long lo = (static_cast<long long>(gw) * W) / p.nwt;
  const long long hi = (static_cast<long long>(gw + 1) * W) / p.nwt;
  if (lane == 0) p.desc[gw] = make_int4(-1, 0, 0, 0);
  if (lo >= hi) return;

  // ---- locate the item `lo`: chunk by binary search, then a warp-wide walk ----
  Cursor<BS> cur;
  cur.k = -1;
  {
    int a = 0, bnd = C::NT - 1;
    while (a < bnd) {  // largest t with scan[t] <= lo
      int m = (a + bnd + 1) >> 1;
      if (scan[m] <= lo) a = m;
      else bnd = m - 1;
    }
    const int s_lo = static_cast<int>((static_cast<long long>(a) * p.S) / C::NT);
    const int s_hi = static_cast<int>((static_cast<long long>(a + 1) * p.S) / C::NT);
    long long base = scan[a];
    for (int s0 = s_lo; s0 < s_hi; s0 += 32) {
      const int s = s0 + lane;
      int len = 0;
      long long w = 0;
      if (s < s_hi) {
        len = __ldg(p.lens + s);
        len = len < 0 ? 0 : (len > max_len ? max_len : len);
        w = static_cast<long long>(p.Hk) * items_of<BS>(len);
      }
      long long incl = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, s < s_hi && base + incl > lo);
      if (hit) {
        const int j = __ffs(hit) - 1;
        const long long start = __shfl_sync(0xffffffffu, base + incl - w, j);
        const int L = __shfl_sync(0xffffffffu, len, j);
        const int n = items_of<BS>(L);
        const long long off = lo - start;
        cur.k = lo;
        cur.s = s0 + j;
        cur.h = static_cast<int>(off / n);
        cur.b = static_cast<int>(off % n);
        cur.L = L;
        cur.n = n;
        break;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (cur.k != lo) {  // unreachable when the scan is consistent; never index with garbage
    if (lane == 0) atomicOr(p.err, kErrBadLen);
    return;
  }

  const uint64_t policy = l2_policy_evict_first();
  const uint32_t my_stages = stages + warp * NS * C::STAGE;
  const uint32_t my_bars = bars + warp * NS * 8;

  // Table-entry window of the producer: lane j holds table[tw_s][tw_b0 + j].
  int tw_s = -1, tw_b0 = 0, tw_val = 0;
  Cursor<BS> pc = cur;

  auto issue = [&](int stage) {
    const uint32_t bar = my_bars + stage * 8;
    if (pc.L == 0) {
      if (lane == 0) mbar_arrive(bar);
      return;
    }
    if (pc.s != tw_s || pc.b < tw_b0 || pc.b >= tw_b0 + 32) {
      tw_s = pc.s;
      tw_b0 = pc.b;
      const int nb = (pc.L + BS - 1) / BS;
      tw_val = (tw_b0 + lane < nb) ? __ldg(p.tables + pc.s * p.t_s + tw_b0 + lane) : 0;
    }
    int phys = __shfl_sync(0xffffffffu, tw_val, pc.b - tw_b0);
    if (phys < 0 || phys >= p.NB) {
      if (lane == 0) atomicOr(p.err, kErrBadBlock);
      phys = 0;
    }
    if (lane == 0) {
      const uint32_t dk = my_stages + stage * C::STAGE;
      const uint32_t dv = dk + C::TILE;
      mbar_arrive_expect_tx(bar, C::STAGE);
#pragma unroll
      for (int hh = 0; hh < C::NH; ++hh)
        tma_load_4d(dk + hh * BS * 128, &p.tmk, bar, hh * C::EPR, 0, pc.h, phys, policy);
#pragma unroll
      for (int hh = 0; hh < C::NH; ++hh)
        tma_load_4d(dv + hh * BS * 128, &p.tmv, bar, hh * C::EPR, 0, pc.h, phys, policy);
    }
  };

  long long issued = 0;
  for (int i = 0; i < NS && pc.k < hi; ++i) {
    issue(i);
    pc.advance(p, max_len);
    ++issued;
  }

  // ---- per-unit state ----
  uint32_t qb[C::KS][2];
  float acc[C::MT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float sl = p.scale_log2;

  const bool h0_ok = (2 * c) < p.g;
  const bool h1_ok = (2 * c + 1) < p.g;

  auto begin_unit = [&]() {
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
    sl = p.scale_log2;
    if constexpr (FP8) sl *= __ldg(p.k_scale + cur.h);
    const bool row_ok = r < p.g;
    const long long qoff = cur.s * p.q_s + (static_cast<long long>(cur.h) * p.g + r) * p.q_h;
    if constexpr (!FP8) {
      const uint32_t* qp = reinterpret_cast<const uint32_t*>(
          static_cast<const uint16_t*>(p.q) + qoff);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        qb[ks][0] = row_ok ? __ldg(qp + (ks * 16 + 2 * c) / 2) : 0u;
        qb[ks][1] = row_ok ? __ldg(qp + (ks * 16 + 8 + 2 * c) / 2) : 0u;
      }
    } else {
      // k-slot order of the widened fp8 tile: slots 2c, 2c+1 <- dims 4c, 4c+1
      // and slots 2c+8, 2c+9 <- dims 4c+2, 4c+3 of each 16-dim step.
      const uint2* qp = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.q) + qoff);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        uint2 v = row_ok ? __ldg(qp + (ks * 16 + 4 * c) / 4) : make_uint2(0u, 0u);
        float f0, f1, f2, f3;
        if constexpr (QBF) {
          f0 = __uint_as_float(v.x << 16);
          f1 = __uint_as_float(v.x & 0xffff0000u);
          f2 = __uint_as_float(v.y << 16);
          f3 = __uint_as_float(v.y & 0xffff0000u);
        } else {
          __half2 a = *reinterpret_cast<__half2*>(&v.x);
          __half2 b = *reinterpret_cast<__half2*>(&v.y);
          f0 = __low2float(a);
          f1 = __high2float(a);
          f2 = __low2float(b);
          f3 = __high2float(b);
        }
        qb[ks][0] = pack2<false>(f0, f1);
        qb[ks][1] = pack2<false>(f2, f3);
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
    if (ub >= lo && ue <= hi) {  // whole unit in this warp: final output
      const float i0 = l0 > 0.f ? vs / l0 : 0.f;
      const float i1 = l1 > 0.f ? vs / l1 : 0.f;
      uint16_t* o = static_cast<uint16_t*>(p.out) + cur.s * p.o_s;
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
        const int db = FP8 ? da + 1 : da + 8;
        if (h0_ok) {
          uint16_t* oh = o + hq0 * p.o_h;
          float x = acc[mt][0] * i0, y = acc[mt][2] * i0;
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
          float x = acc[mt][1] * i1, y = acc[mt][3] * i1;
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
      const long long base = (static_cast<long long>(gw) * 2 + slot) * p.g;
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
        p.desc[gw] = make_int4(cur.s, cur.h, static_cast<int>(ue & 0xffffffffll),
                               static_cast<int>(ue >> 32));
    }
  };

  // ---- main loop ----
  long long it = 0;
  while (cur.k < hi) {
    if (cur.b == 0 || cur.k == lo) begin_unit();
    const int stage = static_cast<int>(it % NS);
    const uint32_t parity = static_cast<uint32_t>((it / NS) & 1);
    if (!warp_wait(my_bars + stage * 8, parity, kWaitNs)) {
      if (lane == 0) atomicOr(p.err, kErrWaitTimeout);
      for (long long j = it + 1; j < issued; ++j)  // let copies in flight land
        warp_wait(my_bars + static_cast<int>(j % NS) * 8, static_cast<uint32_t>((j / NS) & 1),
                  100000000ull);
      return;
    }

    if (cur.L > 0) {
      const uint32_t tk = my_stages + stage * C::STAGE;
      const uint32_t tv = tk + C::TILE;
      const int nvalid = min(BS, cur.L - cur.b * BS);

      // S^T = K Q^T
      float sacc[C::TT][4];
#pragma unroll
      for (int tt = 0; tt < C::TT; ++tt) {
        sacc[tt][0] = sacc[tt][1] = sacc[tt][2] = sacc[tt][3] = 0.f;
        const int trow = tt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        if constexpr (!FP8) {
#pragma unroll
          for (int ks = 0; ks < C::KS; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(tk + swz<BS>(trow, ks * 32 + (lane >> 4) * 16), a0, a1, a2, a3);
            mma16816<MBF>(sacc[tt], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
          }
        } else {
#pragma unroll
          for (int kp = 0; kp < C::KS / 2; ++kp) {
            uint32_t x0, x1, x2, x3;
            ldsm_x4(tk + swz<BS>(trow, kp * 32 + (lane >> 4) * 16), x0, x1, x2, x3);
            mma16816<false>(sacc[tt], e4m3x2_to_f16x2(x0 & 0xffff), e4m3x2_to_f16x2(x1 & 0xffff),
                            e4m3x2_to_f16x2(x0 >> 16), e4m3x2_to_f16x2(x1 >> 16), qb[2 * kp][0],
                            qb[2 * kp][1]);
            mma16816<false>(sacc[tt], e4m3x2_to_f16x2(x2 & 0xffff), e4m3x2_to_f16x2(x3 & 0xffff),
                            e4m3x2_to_f16x2(x2 >> 16), e4m3x2_to_f16x2(x3 >> 16),
                            qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
          }
        }
      }

      // online softmax over this block's tokens, per head column
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int tt = 0; tt < C::TT; ++tt) {
        const int t0 = tt * 16 + r, t1 = t0 + 8;
        sacc[tt][0] = t0 < nvalid ? sacc[tt][0] * sl : -INFINITY;
        sacc[tt][1] = t0 < nvalid ? sacc[tt][1] * sl : -INFINITY;
        sacc[tt][2] = t1 < nvalid ? sacc[tt][2] * sl : -INFINITY;
        sacc[tt][3] = t1 < nvalid ? sacc[tt][3] * sl : -INFINITY;
        mx0 = fmaxf(mx0, fmaxf(sacc[tt][0], sacc[tt][2]));
        mx1 = fmaxf(mx1, fmaxf(sacc[tt][1], sacc[tt][3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: nvalid >= 1
      const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      uint32_t pb[C::TT][2];
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int tt = 0; tt < C::TT; ++tt) {
        const float p0 = exp2f(sacc[tt][0] - mn0), p1 = exp2f(sacc[tt][1] - mn1);
        const float p2 = exp2f(sacc[tt][2] - mn0), p3 = exp2f(sacc[tt][3] - mn1);
        ps0 += p0 + p2;
        ps1 += p1 + p3;
        pb[tt][0] = movmatrix_t(pack2<MBF>(p0, p1));
        pb[tt][1] = movmatrix_t(pack2<MBF>(p2, p3));
      }
      l0 = l0 * al0 + ps0;
      l1 = l1 * al1 + ps1;
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        acc[mt][0] *= al0;
        acc[mt][1] *= al1;
        acc[mt][2] *= al0;
        acc[mt][3] *= al1;
      }

      // O^T += V^T P^T
#pragma unroll
      for (int tt = 0; tt < C::TT; ++tt) {
        // tokens of this thread's A-fragment halves: lo = 2c, hi = 2c+1 (+8 for a2/a3)
        const int tb = tt * 16 + 2 * c;
        const uint32_t keep01 = (tb < nvalid ? 0x0000ffffu : 0u) | (tb + 1 < nvalid ? 0xffff0000u : 0u);
        const uint32_t keep23 =
            (tb + 8 < nvalid ? 0x0000ffffu : 0u) | (tb + 9 < nvalid ? 0xffff0000u : 0u);
        if constexpr (!FP8) {
          const int vrow = tt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
#pragma unroll
          for (int mt = 0; mt < C::MT; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(tv + swz<BS>(vrow, mt * 32 + ((lane >> 3) & 1) * 16), a0, a1, a2, a3);
            mma16816<MBF>(acc[mt], a0 & keep01, a1 & keep01, a2 & keep23, a3 & keep23, pb[tt][0],
                          pb[tt][1]);
          }
        } else {
          const int vrow = tt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int mp = 0; mp < C::MT / 2; ++mp) {
            uint32_t x0, x1, x2, x3;
            ldsm_x4_t(tv + swz<BS>(vrow, mp * 32 + (lane >> 4) * 16), x0, x1, x2, x3);
            const uint32_t e0 = prmt(x0, 0, 0x3120), e1 = prmt(x1, 0, 0x3120);
            const uint32_t e2 = prmt(x2, 0, 0x3120), e3 = prmt(x3, 0, 0x3120);
            mma16816<false>(acc[2 * mp], e4m3x2_to_f16x2(e0 & 0xffff) & keep01,
                            e4m3x2_to_f16x2(e0 >> 16) & keep01,
                            e4m3x2_to_f16x2(e1 & 0xffff) & keep23,
                            e4m3x2_to_f16x2(e1 >> 16) & keep23, pb[tt][0], pb[tt][1]);
            mma16816<false>(acc[2 * mp + 1], e4m3x2_to_f16x2(e2 & 0xffff) & keep01,
                            e4m3x2_to_f16x2(e2 >> 16) & keep01,
                            e4m3x2_to_f16x2(e3 & 0xffff) & keep23,
                            e4m3x2_to_f16x2(e3 >> 16) & keep23, pb[tt][0], pb[tt][1]);
          }
        }
      }
    }

    __syncwarp();
    if (pc.k < hi) {  // refill this stage NS items ahead
      issue(stage);
      pc.advance(p, max_len);
      ++issued;
    }
    if (cur.b == cur.n - 1 || cur.k == hi - 1) finish_unit();
    cur.advance(p, max_len);
    ++it;
  }
}

// Combine the pieces of every unit cut by warp-range boundaries. One CTA per
// warp of the decode grid; the CTA whose warp holds the first piece of a cut
// unit (its slot-1 partial) merges it with the slot-0 partials of the
// following warps whose ranges intersect the unit.
template <bool QBF, int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const __grid_constant__ DecodeParams p) {
  const int gw = blockIdx.x;
  const int4 d = p.desc[gw];
  if (d.x < 0) return;
  const int s = d.x, h = d.y;
  const long long U1 = static_cast<long long>(static_cast<unsigned>(d.z)) |
                       (static_cast<long long>(d.w) << 32);
  const long long W = p.hdr[0];
  const int g = p.g;
  for (int e = threadIdx.x; e < g * D; e += blockDim.x) {
    const int i = e / D, dd = e % D;
    // pass 1: running max over pieces
    float mstar = -INFINITY;
    for (int w = gw;; ++w) {
      const long long lo = (static_cast<long long>(w) * W) / p.nwt;
      if (w > gw && lo >= U1) break;
      const long long hi = (static_cast<long long>(w + 1) * W) / p.nwt;
      if (hi <= lo) continue;
      const int slot = (w == gw) ? 1 : 0;
      mstar = fmaxf(mstar, p.part_ml[((static_cast<long long>(w) * 2 + slot) * g + i) * 2]);
    }
    float lsum = 0.f, osum = 0.f;
    for (int w = gw;; ++w) {
      const long long lo = (static_cast<long long>(w) * W) / p.nwt;
      if (w > gw && lo >= U1) break;
      const long long hi = (static_cast<long long>(w + 1) * W) / p.nwt;
      if (hi <= lo) continue;
      const int slot = (w == gw) ? 1 : 0;
      const long long base = (static_cast<long long>(w) * 2 + slot) * g + i;
      const float mp = p.part_ml[base * 2];
      const float sc = (mp == -INFINITY) ? 0.f : exp2f(mp - mstar);
      lsum += p.part_ml[base * 2 + 1] * sc;
      osum += p.part_o[base * D + dd] * sc;
    }
    const float v = lsum > 0.f ? osum / lsum : 0.f;
    uint16_t* o = static_cast<uint16_t*>(p.out) + s * p.o_s + (static_cast<long long>(h) * g + i) * p.o_h;
    if constexpr (QBF) o[dd] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    else o[dd] = __half_as_ushort(__float2half_rn(v));
  }
}

}  // namespace pkv
