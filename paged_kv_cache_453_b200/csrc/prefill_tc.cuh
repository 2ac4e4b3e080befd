// Multi-token (causal) paged attention on the 5th-generation tensor cores
// (tcgen05 MMAs, accumulators in tensor memory) for wide query tiles: a
// prompt chunk of many new tokens is a dense contraction, so both products
// run as 128 x 128 x 16 tcgen05.mma instructions issued by one thread.
// The result is the one prefill_kernel computes (same positions, same causal
// rule); this kernel is used when a (sequence, kv head) has at least 128
// query rows (new tokens x query heads of the group).
//
// CTA = 8 warps, one (sequence, kv head, 128 query rows); a row is one query
// head of one new token (token-major). Threads r and r + 128 share row r
// (tensor-memory lane r; warps w and w + 4 read the same lane quarter), each
// owning 64 of the 128 columns of S and of O. Per step of 128 keys (128 / B
// blocks through the block table):
//   TMA: the blocks' K and V tiles into a two-stage ring, laid out as two
//        64-column halves of [128 keys x 128 B], 128-byte swizzled
//   S = Q K^T   8 MMAs (K = 16 each) into tensor-memory columns [0, 128)
//   softmax     each thread loads its 64 columns of S once (kept in
//               registers), masks keys past its position, exchanges its
//               max with the row's other thread, runs the online max / sum
//               in the exp2 domain (sums kept per half, added at the end),
//               rescales its half of O in tensor memory and writes its half
//               of P (16-bit) to shared memory in the MMA's layout
//   O += P V    8 MMAs into tensor-memory columns [128, 256), V read as an
//               MN-major operand straight from the TMA tiles
// Loads run two steps ahead; S of the next step is issued as soon as this
// step's S is complete (it runs while this step is reduced: two S buffers in
// tensor memory), and O += P V overlaps the next step's max. Q rows are
// loaded once into shared memory. Shared memory: Q 32 KB, K 2 x 32 KB,
// V 2 x 32 KB, P 32 KB (one CTA per SM); tensor memory: 512 columns.
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

template <int BS>
struct PrefillTcCfg {
  static constexpr int D = 128;
  static constexpr int ROWS = 128;        // query rows per CTA
  static constexpr int KEYS = 128;        // keys per step
  static constexpr int HALF = 128 * 128;  // bytes of a [128 x 64] 16-bit half tile
  static constexpr int TILE = 2 * HALF;   // Q, K, V or P tile: 32 KB
  static constexpr int BPS = KEYS / BS;   // blocks per step
  // layout from the 1024-aligned base: Q | K0 K1 | V0 V1 | P | barriers | tmem slot
  static constexpr int OFF_Q = 0, OFF_K = TILE, OFF_V = 3 * TILE, OFF_P = 5 * TILE;
  static constexpr int OFF_BAR = 6 * TILE;
  static constexpr int OFF_X = OFF_BAR + 128;  // [256] floats: row max / sum exchange
  static constexpr int OFF_PH = OFF_X + 256 * 4;  // [4][BPS] physical blocks, steps mod 4
  static constexpr int SMEM = 1024 + 6 * TILE + 128 + 256 * 4 + 4 * BPS * 4;
};

template <bool QBF, int BS>
__global__ void __launch_bounds__(256, 1) prefill_tc_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillTcCfg<BS>;
  constexpr uint64_t kWaitNs = 2000000000ull;
  // tensor-memory columns: S of even steps [0, 128), of odd steps [128, 256),
  // O [256, 384)
  constexpr uint32_t kCols = 512;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_addr(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - sraw);
  const uint32_t sQ = sbase + C::OFF_Q, sP = sbase + C::OFF_P;
  const uint32_t bar_k = sbase + C::OFF_BAR;  // [2]: K tile of the stage landed
  const uint32_t bar_v = bar_k + 16;          // [2]: V tile of the stage landed
  const uint32_t bar_s = bar_k + 32;          // S of the next step complete
  const uint32_t bar_o = bar_k + 40;          // O += P V complete
  const uint32_t tslot = bar_k + 48;          // tensor-memory base address
  uint32_t* tslot_gen = reinterpret_cast<uint32_t*>(sgen + C::OFF_BAR + 48);
  float* xch = reinterpret_cast<float*>(sgen + C::OFF_X);
  int* s_phys = reinterpret_cast<int*>(sgen + C::OFF_PH);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int rl = tid & 127, half = tid >> 7;  // row in the tile, column half
  const int s = static_cast<int>(blockIdx.z / p.Hk), h = static_cast<int>(blockIdx.z % p.Hk);

  pdl_launch_dependents();
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_k + i * 8, 1);
      mbar_init(bar_v + i * 8, 1);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
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
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tslot_gen);
  const uint32_t tO = tmem + 256;
  const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;  // this warp's lane quarter
  const uint32_t col_off = static_cast<uint32_t>(half * 64);               // this thread's columns

  pdl_wait();
  bool ok = s < p.S;
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
    if (warp == 0) tmem_dealloc(tmem, kCols);
    return;
  }
  const int rend = min(rows_all, r0 + C::ROWS);
  const int lim_max = L - n + (rend - 1) / p.g;
  const int nblk = lim_max / BS + 1;            // blocks any row of the CTA needs
  const int nsteps = (nblk + C::BPS - 1) / C::BPS;

  // this thread's row: its position, or the CTA's last for padding rows
  const int row = r0 + rl;
  const bool row_ok = row < rows_all;
  const int pos = row_ok ? L - n + row / p.g : lim_max;

  // ---- Q row into shared memory (K-major, 128-byte swizzle) ----
  {
    const uint4* qp = reinterpret_cast<const uint4*>(
        static_cast<const uint16_t*>(p.q) + (q0 + (row_ok ? row / p.g : 0)) * p.q_t +
        (static_cast<long long>(h) * p.g + (row_ok ? row % p.g : 0)) * p.q_h);
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {  // this thread's half of the row: chunks 8 half ..
      const int c = half * 8 + cc;
      const uint4 v = row_ok ? __ldg(qp + c) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t a = sQ + (c >> 3) * C::HALF + (rl >> 3) * 1024 + (rl & 7) * 128 +
                         (((c & 7) ^ (rl & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                   "r"(v.w)
                   : "memory");
    }
  }

  // ---- K or V tiles of step i into stage i & 1 (thread 0) ----
  const int* trow = p.tables + s * p.t_s;
  const uint64_t policy = l2_policy_evict_normal();
  // Physical blocks of step i, checked, into s_phys[i % 4] (threads 32 ..
  // 32 + BPS - 1, three steps ahead of their use). Blocks past the ones
  // needed repeat the last needed one (finite data, masked by position).
  auto stage_phys = [&](int i) {
    const int ib = tid - 32;
    if (ib >= 0 && ib < C::BPS && i < nsteps) {
      const int b = min(i * C::BPS + ib, nblk - 1);
      int phys = __ldg(trow + b);
      if (phys < 0 || phys >= p.NB) {
        atomicOr(p.err, kErrBadBlock);
        phys = 0;
      }
      s_phys[(i & 3) * C::BPS + ib] = phys;
    }
  };
  auto issue = [&](int i, bool v_tile) {
    const int st = i & 1;
    const uint32_t bar = (v_tile ? bar_v : bar_k) + st * 8;
    const uint32_t dst = sbase + (v_tile ? C::OFF_V : C::OFF_K) + st * C::TILE;
    const CUtensorMap* map = v_tile ? &p.tmv : &p.tmk;
    mbar_arrive_expect_tx(bar, C::TILE);
#pragma unroll
    for (int ib = 0; ib < C::BPS; ++ib) {
      const int phys = s_phys[(i & 3) * C::BPS + ib];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        tma_load_4d(dst + hh * C::HALF + ib * BS * 128, map, bar, hh * 64, 0, h, phys, policy);
    }
  };
  constexpr uint32_t kIdS = idesc_f16<QBF>(false);  // B = K tile, K-major
  constexpr uint32_t kIdO = idesc_f16<QBF>(true);   // B = V tile, MN-major
  // S of step i = Q K_i^T into its tensor-memory buffer (thread 0)
  auto issue_s = [&](int i) {
    const uint32_t dk = sbase + C::OFF_K + (i & 1) * C::TILE;
    const uint32_t tS = tmem + (i & 1) * 128;
    tc_fence_after();
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t off = (ks >> 2) * C::HALF + (ks & 3) * 32;
      tc_mma(tS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(dk + off, 16, 1024), kIdS, ks > 0);
    }
    tc_commit(bar_s);
  };

  // Loads run two steps ahead, S one step ahead of the softmax, and O += P V
  // of a step overlaps the next step's first pass. Thread 0's counts let a
  // failed wait drain what is in flight.
  int k_issued = 0, v_issued = 0, s_issued = 0, o_issued = 0;
  bool failed = false;
  stage_phys(0);
  stage_phys(1);
  stage_phys(2);
  __syncthreads();
  if (tid == 0) {
    issue(0, false);
    issue(0, true);
    k_issued = v_issued = 1;
    if (nsteps > 1) {
      issue(1, false);
      issue(1, true);
      k_issued = v_issued = 2;
    }
  }
  fence_async_smem();  // Q written by the threads, read by the tensor cores
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (lane_wait(bar_k, 0, kWaitNs)) {
      issue_s(0);
      s_issued = 1;
    } else {
      failed = true;
    }
  }
  failed = __syncthreads_or(failed);

  const float sl = p.scale_log2;
  float m_run = -INFINITY, l_run = 0.f;

  // `failed` is only acted on after a CTA-wide OR, and every warp_wait (whose
  // __all_sync needs all 32 lanes) runs unconditionally; after each block only
  // thread 0 runs, __syncwarp reconverges warp 0 before the warp-collective
  // tensor-memory loads.
  for (int i = 0; i < nsteps; ++i) {
    const int st = i & 1;
    const int key0 = i * C::KEYS;
    const uint32_t tS = tmem + st * 128;
    {
      const bool w_ok = warp_wait(bar_s, static_cast<uint32_t>(i & 1), kWaitNs);
      if (__syncthreads_or(failed || !w_ok)) {
        failed = true;
        break;
      }
    }
    tc_fence_after();
    stage_phys(i + 3);  // read from step i + 1 on, after this step's barriers
    // S of the next step while this one is reduced: its K tile has landed
    // (loaded two steps ahead) and its buffer was read one step ago
    if (tid == 0 && i + 1 < nsteps) {
      if (lane_wait(bar_k + ((i + 1) & 1) * 8, static_cast<uint32_t>(((i + 1) >> 1) & 1), kWaitNs)) {
        issue_s(i + 1);
        ++s_issued;
        // this step's K stage is free now (its S is complete): step i + 2's K
        if (i + 2 < nsteps) {
          issue(i + 2, false);
          ++k_issued;
        }
      } else {
        failed = true;
      }
    }
    __syncwarp();
    // this thread's 64 columns of S, once, into registers (masked, scaled)
    float x[64];
    {
      uint32_t v0[32], v1[32];
      tmem_ld32(tS + lane_off + col_off, v0);
      tmem_ld32(tS + lane_off + col_off + 32, v1);
      tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int k0 = key0 + half * 64 + u;
        x[u] = k0 <= pos ? __uint_as_float(v0[u]) * sl : -INFINITY;
        x[32 + u] = k0 + 32 <= pos ? __uint_as_float(v1[u]) * sl : -INFINITY;
      }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int u = 0; u < 64; ++u) mx = fmaxf(mx, x[u]);
    xch[tid] = mx;  // the row's other thread takes the max of both halves
    __syncthreads();
    mx = fmaxf(mx, xch[tid ^ 128]);
    // The exponent base moves only when the row's max grows by more than 8
    // (P then stays below 2^8, exact enough in 16 bits and far from fp32
    // overflow in O and l); otherwise O needs no rescale this step.
    const float m_new = fmaxf(m_run, mx);
    const bool grow = m_new > m_run + 8.f || m_run == -INFINITY;
    const float m_use = grow ? m_new : m_run;
    const float base = m_use == -INFINITY ? 0.f : m_use;
    const float alpha = grow ? exp2f(m_run - base) : 1.f;
    // the previous step's O += P V must be done before O is rescaled and P
    // rewritten; its V stage then takes step i + 1's V
    if (i > 0) {
      const bool w_ok = warp_wait(bar_o, static_cast<uint32_t>((i - 1) & 1), kWaitNs);
      if (__syncthreads_or(failed || !w_ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      if (tid == 0 && i + 1 < nsteps) {
        issue(i + 1, true);
        ++v_issued;
      }
      __syncwarp();
      // tcgen05.ld / st are warp-collective: rescale when any row of the warp
      // needs it (alpha is 1 for the others)
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
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
    }
    // V rows at or past the sequence's length may hold anything (a partly
    // filled last block): zero them, their P is 0 but 0 * NaN is not
    if (key0 + C::KEYS > L) {
      const bool w_ok = warp_wait(bar_v + st * 8, static_cast<uint32_t>((i >> 1) & 1), kWaitNs);
      if (__syncthreads_or(failed || !w_ok)) {
        failed = true;
        break;
      }
      const uint32_t dv = sbase + C::OFF_V + st * C::TILE;
      for (int k = max(L - key0, 0) * 16 + tid; k < C::KEYS * 16; k += 256) {
        const int key = k >> 4, c = k & 15;  // 16-byte chunk c of key row `key`
        const uint32_t a = dv + (c >> 3) * C::HALF + (key >> 3) * 1024 + (key & 7) * 128 + ((c & 7) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
      }
    }
    // P = exp2(x - m) as 16-bit into shared memory (this thread's 64 keys),
    // this half's sum
    float lsum = 0.f;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      uint32_t pk[16];
#pragma unroll
      for (int u = 0; u < 32; u += 2) {
        const float p0 = exp2f(x[32 * j + u] - base), p1 = exp2f(x[32 * j + u + 1] - base);
        lsum += p0 + p1;
        pk[u >> 1] = pack2<QBF>(p0, p1);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // 16-byte chunk 4 j + u of this half of the keys
        const int kc = 4 * j + u;
        const uint32_t a = sP + half * C::HALF + (rl >> 3) * 1024 + (rl & 7) * 128 +
                           (((kc & 7) ^ (rl & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * u]),
                     "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                     : "memory");
      }
    }
    l_run = l_run * alpha + lsum;
    m_run = m_use;
    tmem_wait_st();
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(failed)) {
      failed = true;
      break;
    }
    if (tid == 0) {  // O += P V, once this step's V tile has landed
      if (lane_wait(bar_v + st * 8, static_cast<uint32_t>((i >> 1) & 1), kWaitNs)) {
        tc_fence_after();
        const uint32_t dv = sbase + C::OFF_V + st * C::TILE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t a_off = (ks >> 2) * C::HALF + (ks & 3) * 32;  // keys 16 ks .. of P
          tc_mma(tO, smem_desc_sw128(sP + a_off, 16, 1024),
                 smem_desc_sw128(dv + ks * 2048, C::HALF, 1024), kIdO, (i > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(bar_o);
        ++o_issued;
      } else {
        failed = true;
      }
    }
    __syncwarp();
  }

  failed = __syncthreads_or(failed);
  if (!failed) {
    const bool w_ok = warp_wait(bar_o, static_cast<uint32_t>((nsteps - 1) & 1), kWaitNs);
    failed = __syncthreads_or(!w_ok);
  }
  if (failed) {
    if (tid == 0) {
      atomicOr(p.err, kErrWaitTimeout);
      // let what is still in flight finish (bounded) before the CTA's shared
      // and tensor memory go: every issued load and the last products
      constexpr uint64_t kDrainNs = 100000000ull;
      // loads into one stage complete in order: wait for each stage's last
      for (int k = max(k_issued - 2, 0); k < k_issued; ++k)
        lane_wait(bar_k + (k & 1) * 8, static_cast<uint32_t>((k >> 1) & 1), kDrainNs);
      for (int k = max(v_issued - 2, 0); k < v_issued; ++k)
        lane_wait(bar_v + (k & 1) * 8, static_cast<uint32_t>((k >> 1) & 1), kDrainNs);
      if (s_issued > 0) lane_wait(bar_s, static_cast<uint32_t>((s_issued - 1) & 1), kDrainNs);
      if (o_issued > 0) lane_wait(bar_o, static_cast<uint32_t>((o_issued - 1) & 1), kDrainNs);
    }
  } else {
    tc_fence_after();
    // epilogue: O row / l (both halves' sums), 16-bit, to the output row
    xch[tid] = l_run;
    __syncthreads();
    const float lt = l_run + xch[tid ^ 128];
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}

}  // namespace pkv
