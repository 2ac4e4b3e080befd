// Multi-token (causal) paged attention on the 5th-generation tensor cores
// (tcgen05 MMAs, accumulators in tensor memory) for wide query tiles: a
// prompt chunk of many new tokens is a dense contraction, so both products
// run as 128 x 128 x 16 tcgen05.mma instructions issued by one thread.
// The result is the one prefill_kernel computes (same positions, same causal
// rule); this kernel is used when a (sequence, kv head) may have at least
// 64 query rows (new tokens x query heads of the group).
//
// CTA = 8 softmax warps + 4 producer warps, one (sequence, kv head, 128 query
// rows); a row is one query head of one new token (token-major). Threads r
// and r + 128 share row r (tensor-memory lane r; warps w and w + 4 read the
// same lane quarter), each owning 64 of the 128 columns of S and of O. One
// producer warp issues the MMAs, two the K loads, one the V loads (issuing a
// paged load or an MMA costs far more than its few instructions suggest, so
// they proceed side by side); they and the softmax warps meet only at
// mbarriers (S ready, P ready, O done, stage landed), never at a CTA-wide
// barrier inside the loop. Per step of 128 keys (128 / B blocks through the
// block table):
//   TMA: the blocks' K and V tiles into a two-stage ring, laid out as two
//        64-column halves of [128 keys x 128 B], 128-byte swizzled
//   S = Q K^T   8 MMAs (K = 16 each) into one of two S buffers in tensor
//               memory (columns [0, 128) for even steps, [128, 256) odd)
//   softmax     each thread loads its 64 columns of S once (kept in
//               registers), masks keys past its position, exchanges its
//               max with the row's other thread, runs the online max / sum
//               in the exp2 domain (sums kept per half, added at the end),
//               rescales its half of O in tensor memory and writes its half
//               of P (16-bit) to shared memory in the MMA's layout
//   O += P V    8 MMAs into tensor-memory columns [256, 384), V read as an
//               MN-major operand straight from the TMA tiles
// Loads run up to two steps ahead (a stage is reloaded once the product that
// read it is complete); S of the next step is issued as soon as its K has
// landed, so it runs while this step is reduced. P is double-buffered in shared memory, so a step's softmax
// waits for the previous step's O += P V only when O must be rescaled. Q rows
// are loaded once into shared memory. Shared memory: Q 32 KB, K 2 x 32 KB,
// V 2 x 32 KB, P 2 x 32 KB (one CTA per SM); tensor memory: 512 columns.
#pragma once

#include "prefill.cuh"

namespace pkv {

// ---- tcgen05 / tensor memory helpers ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16, fp32 accumulate
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on an mbarrier once all prior tcgen05.mma of this thread complete
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
      "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a 128-byte-swizzled tile (version 1):
// start address, leading / stride byte offsets (16-byte units).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16, fp32 accumulate, M = 128, N = 128.
template <bool BF16>
__device__ __forceinline__ constexpr uint32_t idesc_f16(bool b_mn_major) {
  return (1u << 4) | ((BF16 ? 1u : 0u) << 7) | ((BF16 ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}

// ---- packed fp32 pairs (two lanes of one 64-bit register) and 3-input max ----
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
template <int BS>
struct PrefillTcCfg {
  static constexpr int D = 128;
  static constexpr int ROWS = 128;        // query rows per CTA
  static constexpr int KEYS = 128;        // keys per step
  static constexpr int HALF = 128 * 128;  // bytes of a [128 x 64] 16-bit half tile
  static constexpr int TILE = 2 * HALF;   // Q, K, V or P tile: 32 KB
  static constexpr int BPS = KEYS / BS;   // blocks per step
  static constexpr int SOFT = 256;        // softmax threads (8 warps)
  static constexpr int LWK = 2, LWV = 1;  // warps loading the K / V tile of a step
  static_assert(BPS % LWK == 0 && BPS % LWV == 0, "a loading warp takes whole blocks");
  // warp 8 issues the MMAs, the next LWK warps load K, the LWV after them V
  static constexpr int THREADS = SOFT + 32 * (1 + LWK + LWV);
  // layout from the (1024-aligned) base:
  //   Q | K0 K1 | V0 V1 | P0 P1 | barriers | exchange | flags
  static constexpr int OFF_Q = 0, OFF_K = TILE, OFF_V = 3 * TILE, OFF_P = 5 * TILE;
  static constexpr int OFF_BAR = 7 * TILE;
  static constexpr int OFF_X = OFF_BAR + 128;     // [2][256] floats: row max / sum exchange
  static constexpr int OFF_F = OFF_X + 512 * 4;   // [2][8] ints: a softmax warp's wait failed
  static constexpr int SMEM = OFF_F + 16 * 4;
  static_assert(SMEM <= 227 * 1024, "more shared memory than a CTA can have");
};

constexpr int kErrTcSetup = 32;  // shared or tensor memory not placed as the kernel assumes

// Named barrier of the two softmax warps that share a lane quarter (w, w + 4).
__device__ __forceinline__ void pair_sync(int quarter) {
  asm volatile("bar.sync %0, 64;" ::"r"(quarter + 1) : "memory");
}

template <bool QBF, int BS>
__global__ void __launch_bounds__(PrefillTcCfg<BS>::THREADS, 1) prefill_tc_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillTcCfg<BS>;
  constexpr uint64_t kWaitNs = 2000000000ull;
  // tensor-memory columns: S of even steps [0, 128), of odd steps [128, 256),
  // O [256, 384)
  constexpr uint32_t kCols = 512;

  // The 128-byte swizzle repeats every 1024 bytes and the tiles' descriptors
  // assume it starts at each tile; the buffer leaves no room to round up.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_addr(smem_raw);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrTcSetup);
    return;
  }
  uint8_t* sgen = smem_raw;
  const uint32_t sQ = sbase + C::OFF_Q, sP = sbase + C::OFF_P;
  const uint32_t bar_k = sbase + C::OFF_BAR;  // [2]: K tile of the stage landed
  const uint32_t bar_v = bar_k + 16;          // [2]: V tile of the stage landed
  // Each barrier's phases are waited in order and never two behind (a phase
  // cannot complete twice before its waiters pass): S has one barrier per
  // tensor-memory buffer, and each wait is placed before the issue that
  // could complete that barrier's next phase.
  const uint32_t bar_s = bar_k + 32;          // [2]: S of the buffer's step complete
  const uint32_t bar_o = bar_k + 48;          // [2]: O += P V of a step complete (by P buffer)
  const uint32_t bar_p = bar_k + 64;          // [2]: P of a step written (softmax threads arrive)
  const uint32_t bar_q = bar_k + 80;          // Q written (softmax threads arrive)
  const uint32_t tslot = bar_k + 88;          // tensor-memory base address
  uint32_t* tslot_gen = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + 88);
  float* xch = reinterpret_cast<float*>(sgen + C::OFF_X);
  int* xfail = reinterpret_cast<int*>(sgen + C::OFF_F);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rl = tid & 127, half = (tid >> 7) & 1;  // softmax: row in the tile, column half
  const int zs = static_cast<int>(blockIdx.z / p.Hk), h = static_cast<int>(blockIdx.z % p.Hk);

  pdl_launch_dependents();
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_k + i * 8, C::LWK);
      mbar_init(bar_v + i * 8, C::LWV);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_s + 8, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_o + 8, 1);
    mbar_init(bar_p, C::SOFT);
    mbar_init(bar_p + 8, C::SOFT);
    mbar_init(bar_q, C::SOFT);
    tma_prefetch_desc(&p.tmk);
    tma_prefetch_desc(&p.tmv);
  }
  fence_mbar_init();
  if (warp == 0) {
    tmem_alloc(tslot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // A 512-column allocation is the whole tensor memory, so it starts at lane
  // 0, column 0; the constant keeps the MMA operands in uniform registers.
  const uint32_t tmem_got = *reinterpret_cast<volatile uint32_t*>(tslot_gen);
  constexpr uint32_t tmem = 0;
  constexpr uint32_t tO = tmem + 256;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;  // this warp's lane quarter
  const uint32_t col_off = static_cast<uint32_t>(half * 64);               // this thread's columns

  pdl_wait();
  // the sequence: in launch order, or longest context first when an order
  // was computed (it shortens the tail of the last wave)
  const int s = p.order ? p.order[zs] : zs;
  bool ok = s >= 0 && s < p.S;
  if (tmem_got != tmem) {
    if (tid == 0) atomicOr(p.err, kErrTcSetup);
    ok = false;
  }
  int q0 = 0, n = 0, L = 0;
  if (ok) {
    q0 = __ldg(p.q_start + s);
    const int q1 = __ldg(p.q_start + s + 1);
    L = __ldg(p.lens + s);
    n = q1 - q0;
    if (n < 0 || L < n || L > p.MB * BS || q0 < 0 || q1 > p.T) {
      if (tid == 0 && blockIdx.x == 0) atomicOr(p.err, kErrBadLen);
      ok = false;
    }
  }
  const int rows_all = n * p.g;
  const int r0 = blockIdx.x * C::ROWS;  // first query row of this CTA
  if (tid == 0 && ok && blockIdx.x == 0 && rows_all > static_cast<int>(gridDim.x) * C::ROWS)
    atomicOr(p.err, kErrBadLen);  // more new tokens than max_q_tokens
  ok = ok && r0 < rows_all;
  if (!ok) {
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem_got, kCols);
    return;
  }
  const int rend = min(rows_all, r0 + C::ROWS);
  const int lim_max = L - n + (rend - 1) / p.g;
  const int nblk = lim_max / BS + 1;            // blocks any row of the CTA needs
  const int nsteps = (nblk + C::BPS - 1) / C::BPS;
  int* err = p.err;

  if (warp >= C::SOFT / 32) {
    // ================= producer warps =================
    bool ok_p = true;
    auto wait1 = [&](uint32_t bar, uint32_t parity) {  // lane 0 waits, the warp learns
      bool w = true;
      if (lane == 0) w = lane_wait(bar, parity, kWaitNs);
      w = __shfl_sync(0xffffffffu, w, 0);
      ok_p = ok_p && w;
      return w;
    };
    constexpr uint64_t kDrainNs = 100000000ull;
    if (warp == C::SOFT / 32) {
      // ---- MMA issue: S of step i + 1 before O += P V of step i ----
      constexpr uint32_t kIdS = idesc_f16<QBF>(false);  // B = K tile, K-major
      constexpr uint32_t kIdO = idesc_f16<QBF>(true);   // B = V tile, MN-major
      // descriptors of each operand's stage 0; a stage or a K step moves the
      // start address field (16-byte units, no carry: shared addresses are
      // below 256 KB)
      const uint64_t d_q = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t d_k = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t d_p = smem_desc_sw128(sP, 16, 1024);
      const uint64_t d_v = smem_desc_sw128(sbase + C::OFF_V, C::HALF, 1024);
      auto issue_s = [&](int i) {  // lane 0: S of step i into its buffer
        const uint64_t dk = d_k + static_cast<uint64_t>((i & 1) * (C::TILE >> 4));
        const uint32_t tS = tmem + (i & 1) * 128;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          constexpr int kHalf16 = C::HALF >> 4;
          const uint64_t off = static_cast<uint64_t>((ks >> 2) * kHalf16 + (ks & 3) * 2);
          tc_mma(tS, d_q + off, dk + off, kIdS, ks > 0);
        }
        tc_commit(bar_s + (i & 1) * 8);
      };
      auto issue_pv = [&](int i) {  // lane 0: O += P V of step i
        const uint64_t dv = d_v + static_cast<uint64_t>((i & 1) * (C::TILE >> 4));
        const uint64_t dp = d_p + static_cast<uint64_t>((i & 1) * (C::TILE >> 4));
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          constexpr int kHalf16 = C::HALF >> 4;
          const uint64_t a_off = static_cast<uint64_t>((ks >> 2) * kHalf16 + (ks & 3) * 2);  // keys 16 ks ..
          tc_mma(tO, dp + a_off, dv + static_cast<uint64_t>(ks * (2048 >> 4)), kIdO, (i > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(bar_o + (i & 1) * 8);
      };
      int s_issued = 0, o_issued = 0;
      if (wait1(bar_q, 0) && wait1(bar_k, 0)) {
        if (lane == 0) issue_s(0);
        s_issued = 1;
      }
      for (int i = 0; i < nsteps && ok_p; ++i) {
        // S of step i + 1 while step i is reduced: its K has landed; its
        // buffer was last read by step i - 1's softmax, whose P was awaited
        // below one step ago
        if (i + 1 < nsteps) {
          if (!wait1(bar_k + ((i + 1) & 1) * 8, static_cast<uint32_t>(((i + 1) >> 1) & 1))) break;
          if (lane == 0) issue_s(i + 1);
          ++s_issued;
        }
        // O += P V of step i once its P is written and its V landed
        if (!wait1(bar_p + (i & 1) * 8, static_cast<uint32_t>((i >> 1) & 1))) break;
        if (!wait1(bar_v + (i & 1) * 8, static_cast<uint32_t>((i >> 1) & 1))) break;
        if (lane == 0) issue_pv(i);
        ++o_issued;
        __syncwarp();
      }
      if (lane == 0) {
        if (!ok_p) atomicOr(err, kErrWaitTimeout);
        // the last products complete before the CTA leaves (at once unless a
        // wait ran out somewhere)
        for (int k = max(s_issued - 2, 0); k < s_issued; ++k)
          lane_wait(bar_s + (k & 1) * 8, static_cast<uint32_t>((k >> 1) & 1), kDrainNs);
        for (int k = max(o_issued - 2, 0); k < o_issued; ++k)
          lane_wait(bar_o + (k & 1) * 8, static_cast<uint32_t>((k >> 1) & 1), kDrainNs);
      }
    } else {
      // ---- K or V tiles of each step, two stages; LWK (LWV) warps per tile,
      // each loading an equal share of the step's blocks ----
      // A stage is free again once the product that read it (S, or O += P V,
      // of two steps before) is complete. Lanes 0 .. BPS - 1 hold the step's
      // physical blocks (read a step ahead); blocks past the ones needed
      // repeat the last needed one (finite data, masked).
      const int lw = warp - C::SOFT / 32 - 1;  // 0 .. LWK + LWV - 1
      const bool vt = lw >= C::LWK;
      const int nlw = vt ? C::LWV : C::LWK;
      const int nb = C::BPS / nlw;  // blocks this warp loads
      const int ib0 = (vt ? lw - C::LWK : lw) * nb;
      const int* trow = p.tables + s * p.t_s;
      const uint64_t policy = l2_policy_evict_normal();
      const uint32_t full = vt ? bar_v : bar_k;
      const uint32_t done = vt ? bar_o : bar_s;
      const CUtensorMap* map = vt ? &p.tmv : &p.tmk;
      const uint32_t dst0 = sbase + (vt ? C::OFF_V : C::OFF_K);
      auto load_phys = [&](int j) {
        return lane < C::BPS && j < nsteps ? __ldg(trow + min(j * C::BPS + lane, nblk - 1)) : 0;
      };
      int phys = load_phys(0);
      int issued = 0;
      for (int j = 0; j < nsteps; ++j) {
        const int phys_next = load_phys(j + 1);
        if (lane < C::BPS && (phys < 0 || phys >= p.NB)) {
          atomicOr(err, kErrBadBlock);
          phys = 0;
        }
        if (j >= 2 && !wait1(done + (j & 1) * 8, static_cast<uint32_t>(((j - 2) >> 1) & 1))) break;
        const uint32_t bar = full + (j & 1) * 8, dst = dst0 + (j & 1) * C::TILE;
        int pb[C::BPS];
#pragma unroll
        for (int u = 0; u < C::BPS; ++u) pb[u] = __shfl_sync(0xffffffffu, phys, min(ib0 + u, C::BPS - 1));
        if (lane == 0) {
          mbar_arrive_expect_tx(bar, C::TILE / nlw);
#pragma unroll
          for (int u = 0; u < C::BPS; ++u)
            if (u < nb) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh)
                tma_load_4d(dst + hh * C::HALF + (ib0 + u) * BS * 128, map, bar, hh * 64, 0, h, pb[u], policy);
            }
        }
        ++issued;
        phys = phys_next;
      }
      if (lane == 0) {
        if (!ok_p) atomicOr(err, kErrWaitTimeout);
        // the last loads land before the CTA's shared memory is released
        for (int k = max(issued - 2, 0); k < issued; ++k)
          lane_wait(full + (k & 1) * 8, static_cast<uint32_t>((k >> 1) & 1), kDrainNs);
      }
    }
    __syncwarp();
  } else {
    // ================= softmax warps =================
    const int quarter = warp & 3;
    const int row = r0 + rl;
    const bool row_ok = row < rows_all;
    const int pos = row_ok ? L - n + row / p.g : lim_max;  // padding rows: the CTA's last
    // Q row half into shared memory (K-major, 128-byte swizzle)
    {
      const uint4* qp = reinterpret_cast<const uint4*>(
          static_cast<const uint16_t*>(p.q) + (q0 + (row_ok ? row / p.g : 0)) * p.q_t +
          (static_cast<long long>(h) * p.g + (row_ok ? row % p.g : 0)) * p.q_h);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const int c = half * 8 + cc;
        const uint4 v = row_ok ? __ldg(qp + c) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t a = sQ + (c >> 3) * C::HALF + (rl >> 3) * 1024 + (rl & 7) * 128 +
                           (((c & 7) ^ (rl & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                     "r"(v.w)
                     : "memory");
      }
      fence_async_smem();  // Q written by the threads, read by the tensor cores
      mbar_arrive(bar_q);
    }
    const float sl = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok_s = true;
    int xs = 0;  // exchange slot: alternates, so a thread never overwrites a value its partner has yet to read
    for (int i = 0; i < nsteps; ++i) {
      const int key0 = i * C::KEYS;
      const uint32_t tS = tmem + (i & 1) * 128;
      // The waits of a step come before the pair's exchange, so both warps of
      // the pair learn there whether either gave up (here or in the previous
      // step's rescale) and leave together: the named barrier has no time limit.
      bool w = ok_s && warp_wait(bar_s + (i & 1) * 8, static_cast<uint32_t>((i >> 1) & 1), kWaitNs);
      // this thread's 64 columns of S, once, into registers: raw scores (the
      // scale is applied inside the exponent; it is positive), keys past the
      // row's position set to -inf (only in steps where the warp has any)
      float x[64];
      float mx = -INFINITY;
      if (w) {
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tS + lane_off + col_off, v0);
        tmem_ld32(tS + lane_off + col_off + 32, v1);
        tmem_wait_ld();
        const int kfirst = key0 + half * 64;
        if (__any_sync(0xffffffffu, kfirst + 63 > pos)) {
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            x[u] = kfirst + u <= pos ? __uint_as_float(v0[u]) : -INFINITY;
            x[32 + u] = kfirst + 32 + u <= pos ? __uint_as_float(v1[u]) : -INFINITY;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            x[u] = __uint_as_float(v0[u]);
            x[32 + u] = __uint_as_float(v1[u]);
          }
        }
        float mm[4];  // four independent chains of 16
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          mm[c] = fmax3(x[16 * c], x[16 * c + 1], x[16 * c + 2]);
#pragma unroll
          for (int u = 3; u < 15; u += 2) mm[c] = fmax3(mm[c], x[16 * c + u], x[16 * c + u + 1]);
          mm[c] = fmaxf(mm[c], x[16 * c + 15]);
        }
        mx = fmaxf(fmax3(mm[0], mm[1], mm[2]), mm[3]) * sl;
      }
      // this step's P buffer was last read by step i - 2's O += P V; V rows
      // of this step are zeroed below once they landed
      if (w && i >= 2) w = warp_wait(bar_o + (i & 1) * 8, static_cast<uint32_t>(((i - 2) >> 1) & 1), kWaitNs);
      const bool tail = key0 + C::KEYS > L;
      if (w && tail) w = warp_wait(bar_v + (i & 1) * 8, static_cast<uint32_t>((i >> 1) & 1), kWaitNs);
      xch[xs * 256 + tid] = mx;  // the row's other thread takes the max of both halves
      if (lane == 0) xfail[xs * 8 + warp] = w ? 0 : 1;
      pair_sync(quarter);
      if (xfail[xs * 8 + quarter] | xfail[xs * 8 + quarter + 4]) {
        ok_s = false;
        xs ^= 1;
        break;
      }
      mx = fmaxf(mx, xch[xs * 256 + (tid ^ 128)]);
      xs ^= 1;
      // The exponent base moves only when the row's max grows by more than 8
      // (P then stays below 2^8, exact enough in 16 bits and far from fp32
      // overflow in O and l); otherwise O needs no rescale this step.
      const float m_new = fmaxf(m_run, mx);
      const bool grow = m_new > m_run + 8.f || m_run == -INFINITY;
      const float m_use = grow ? m_new : m_run;
      const float base = m_use == -INFINITY ? 0.f : m_use;
      const float alpha = grow ? exp2f(m_run - base) : 1.f;
      // tcgen05.ld / st are warp-collective: rescale when any row of the warp
      // needs it (alpha is 1 for the others; both warps of a pair hold the
      // same rows, so they decide alike), once step i - 1's O += P V is complete
      if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f) &&
          (ok_s = warp_wait(bar_o + ((i - 1) & 1) * 8, static_cast<uint32_t>(((i - 1) >> 1) & 1), kWaitNs))) {
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tO + lane_off + col_off, v0);
        tmem_ld32(tO + lane_off + col_off + 32, v1);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          v0[u] = __float_as_uint(__uint_as_float(v0[u]) * alpha);
          v1[u] = __float_as_uint(__uint_as_float(v1[u]) * alpha);
        }
        tmem_st32(tO + lane_off + col_off, v0);
        tmem_st32(tO + lane_off + col_off + 32, v1);
      }
      // V rows at or past the sequence's length may hold anything (a partly
      // filled last block): zero them, their P is 0 but 0 * NaN is not
      if (tail) {
        const uint32_t dv = sbase + C::OFF_V + (i & 1) * C::TILE;
        for (int k = max(L - key0, 0) * 16 + tid; k < C::KEYS * 16; k += C::SOFT) {
          const int key = k >> 4, c = k & 15;  // 16-byte chunk c of key row `key`
          const uint32_t a = dv + (c >> 3) * C::HALF + (key >> 3) * 1024 + (key & 7) * 128 + ((c & 7) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
        }
      }
      // P = 2^(x sl - base) as 16-bit into shared memory (this thread's 64
      // keys); pairs of lanes through the packed fp32 unit
      const uint64_t sl2 = f2_pack(sl, sl), nb2 = f2_pack(-base, -base);
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // partial row sums, pairs
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 32; u += 2) {
          float t0, t1;
          f2_unpack(f2_fma(f2_pack(x[32 * j + u], x[32 * j + u + 1]), sl2, nb2), t0, t1);
          const float p0 = ex2_fast(t0), p1 = ex2_fast(t1);
          acc[(u >> 1) & 3] = f2_add(acc[(u >> 1) & 3], f2_pack(p0, p1));
          pk[u >> 1] = pack2<QBF>(p0, p1);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // 16-byte chunk 4 j + u of this half of the keys
          const int kc = 4 * j + u;
          const uint32_t a = sP + (i & 1) * C::TILE + half * C::HALF + (rl >> 3) * 1024 + (rl & 7) * 128 +
                             (((kc & 7) ^ (rl & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * u]),
                       "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                       : "memory");
        }
      }
      float lsum0, lsum1;
      f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lsum0, lsum1);
      const float lsum = lsum0 + lsum1;
      l_run = l_run * alpha + lsum;
      m_run = m_use;
      tmem_wait_st();
      fence_async_smem();  // P (and zeroed V rows) for the tensor cores
      tc_fence_before();
      mbar_arrive(bar_p + (i & 1) * 8);
    }
    if (ok_s && !warp_wait(bar_o + ((nsteps - 1) & 1) * 8, static_cast<uint32_t>(((nsteps - 1) >> 1) & 1), kWaitNs))
      ok_s = false;
    // epilogue: O row / l (both halves' sums), 16-bit, to the output row
    xch[xs * 256 + tid] = l_run;
    pair_sync(quarter);
    if (ok_s) {
      tc_fence_after();
      const float lt = l_run + xch[xs * 256 + (tid ^ 128)];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      uint4* orow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) +
                                             (q0 + (row_ok ? row / p.g : 0)) * p.o_t +
                                             (static_cast<long long>(h) * p.g + (row_ok ? row % p.g : 0)) * p.o_h +
                                             half * 64);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t v[32];
        tmem_ld32(tO + lane_off + col_off + j * 32, v);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack2<QBF>(__uint_as_float(v[8 * u + 0]) * inv, __uint_as_float(v[8 * u + 1]) * inv);
            w.y = pack2<QBF>(__uint_as_float(v[8 * u + 2]) * inv, __uint_as_float(v[8 * u + 3]) * inv);
            w.z = pack2<QBF>(__uint_as_float(v[8 * u + 4]) * inv, __uint_as_float(v[8 * u + 5]) * inv);
            w.w = pack2<QBF>(__uint_as_float(v[8 * u + 6]) * inv, __uint_as_float(v[8 * u + 7]) * inv);
            orow[4 * j + u] = w;
          }
        }
      }
    } else if (lane == 0) {
      atomicOr(err, kErrWaitTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}

}  // namespace pkv
