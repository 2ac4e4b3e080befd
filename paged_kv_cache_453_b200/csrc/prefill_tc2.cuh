// Multi-token (causal) paged attention on tcgen05, two 128-row query tiles
// per CTA. Same result as prefill_tc_kernel (same positions, same causal
// rule, same lazily moved exponent base); the difference is the schedule.
//
// CTA = 8 softmax warps + 4 producer warps, one (sequence, kv head, 256
// query rows) as two tiles A and B of 128 rows. Warps 0-3 reduce tile A,
// warps 4-7 tile B; a thread owns one row (its tensor-memory lane) and all
// 128 columns of it, so a row needs no exchange between threads. The two
// tiles share every K and V tile of a step, and while one tile's softmax
// runs the tensor core works on the other's products:
//   S_A(0) S_B(0) | pv_A(0) S_A(1) pv_B(0) S_B(1) | pv_A(1) S_A(2) ...
// Tensor memory (512 columns): S_A [0, 128), O_A [128, 256), S_B [256, 384),
// O_B [384, 512). P (16-bit, two per column) is written by the softmax
// threads over the first 64 columns of their tile's S and read from there by
// O += P V as the MMA's A operand; the next S of that tile is issued after
// that product, and tcgen05 MMAs of one thread run in issue order, so S
// overwrites P only after the product has read it. The completion of S_t(i)
// thereby also tells the tile's softmax that O_t += P_t(i - 1) V is done
// (O may be rescaled and P rewritten).
// Producer warps: one issues the MMAs, two load each step's K blocks, one
// its V blocks (TMA, two-stage rings, 128-byte swizzle); a stage is reloaded
// once the step's last S (for K) or last product (for V) has completed.
// Shared memory: Q 2 x 32 KB, K 2 x 32 KB, V 2 x 32 KB.
#pragma once

#include "prefill_tc.cuh"

namespace pkv {

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16, fp32 accumulate: A is M x K
// with row m in lane m, two 16-bit elements of consecutive k per column
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

template <int BS>
struct PrefillTc2Cfg {
  static constexpr int D = 128;
  static constexpr int ROWS = 256;        // query rows per CTA (two tiles)
  static constexpr int KEYS = 128;        // keys per step
  static constexpr int HALF = 128 * 128;  // bytes of a [128 x 64] 16-bit half tile
  static constexpr int TILE = 2 * HALF;   // Q, K or V tile: 32 KB
  static constexpr int BPS = KEYS / BS;   // blocks per step
  static constexpr int LWK = 2, LWV = 1;  // warps loading the K / V tile of a step
  static_assert(BPS % LWK == 0 && BPS % LWV == 0, "a loading warp takes whole blocks");
  static constexpr int SOFT = 256;        // softmax threads: 128 per tile
  static constexpr int THREADS = SOFT + 32 * (1 + LWK + LWV);
  // Q_A Q_B | K0 K1 | V0 V1 | barriers
  static constexpr int OFF_Q = 0, OFF_K = 2 * TILE, OFF_V = 4 * TILE, OFF_BAR = 6 * TILE;
  static constexpr int SMEM = OFF_BAR + 256;
  static_assert(SMEM <= 227 * 1024, "more shared memory than a CTA can have");
};

template <bool QBF, int BS>
__global__ void __launch_bounds__(PrefillTc2Cfg<BS>::THREADS, 1)
    prefill_tc2_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillTc2Cfg<BS>;
  constexpr uint64_t kWaitNs = 2000000000ull;
  constexpr uint64_t kDrainNs = 100000000ull;
  constexpr uint32_t kCols = 512;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t sbase = smem_addr(smem_raw);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicOr(p.err, kErrTcSetup);
    return;
  }
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t bar_k = bar0;         // [2] K tile of the stage landed (LWK arrivals)
  const uint32_t bar_v = bar0 + 16;    // [2] V tile of the stage landed (LWV arrivals)
  const uint32_t bar_kf = bar0 + 32;   // [2] K stage free: the step's last S complete
  const uint32_t bar_vf = bar0 + 48;   // [2] V stage free: the step's last product complete
  const uint32_t bar_s = bar0 + 64;    // [tile] S of the step complete
  const uint32_t bar_p = bar0 + 80;    // [tile] P of the step written (128 arrivals)
  const uint32_t bar_o = bar0 + 96;    // [tile] the last O += P V complete
  const uint32_t bar_q = bar0 + 112;   // Q written (256 arrivals)
  const uint32_t bar_done = bar0 + 120;  // every MMA of the CTA complete
  const uint32_t tslot = bar0 + 128;   // tensor-memory base address
  uint32_t* tslot_gen = reinterpret_cast<uint32_t*>(smem_raw + C::OFF_BAR + 128);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int zs = static_cast<int>(blockIdx.z / p.Hk), h = static_cast<int>(blockIdx.z % p.Hk);

  pdl_launch_dependents();
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_k + i * 8, C::LWK);
      mbar_init(bar_v + i * 8, C::LWV);
      mbar_init(bar_kf + i * 8, 1);
      mbar_init(bar_vf + i * 8, 1);
      mbar_init(bar_s + i * 8, 1);
      mbar_init(bar_p + i * 8, 128);
      mbar_init(bar_o + i * 8, 1);
    }
    mbar_init(bar_q, C::SOFT);
    mbar_init(bar_done, 1);
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
  const int nt = rend - r0 > 128 ? 2 : 1;  // tiles with rows
  const int lim_max = L - n + (rend - 1) / p.g;
  const int nblk = lim_max / BS + 1;  // blocks any row of the CTA needs
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
    if (warp == C::SOFT / 32) {
      // ---- MMA issue ----
      constexpr uint32_t kIdS = idesc_f16<QBF>(false);  // B = K tile, K-major
      constexpr uint32_t kIdO = idesc_f16<QBF>(true);   // B = V tile, MN-major
      constexpr int kHalf16 = C::HALF >> 4;
      const uint64_t d_q = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t d_k = smem_desc_sw128(sbase + C::OFF_K, 16, 1024);
      const uint64_t d_v = smem_desc_sw128(sbase + C::OFF_V, C::HALF, 1024);
      auto issue_s = [&](int t, int i) {  // lane 0: S_t of step i
        const uint64_t dq = d_q + static_cast<uint64_t>(t * (C::TILE >> 4));
        const uint64_t dk = d_k + static_cast<uint64_t>((i & 1) * (C::TILE >> 4));
        const uint32_t tS = tmem + t * 256;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t off = static_cast<uint64_t>((ks >> 2) * kHalf16 + (ks & 3) * 2);
          tc_mma(tS, dq + off, dk + off, kIdS, ks > 0);
        }
        tc_commit(bar_s + t * 8);
      };
      auto issue_pv = [&](int t, int i) {  // lane 0: O_t += P_t V of step i
        const uint64_t dv = d_v + static_cast<uint64_t>((i & 1) * (C::TILE >> 4));
        const uint32_t tS = tmem + t * 256, tO = tS + 128;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // P's keys 16 ks .. in columns 8 ks .. of the tile's S
          tc_mma_ts(tO, tS + 8 * ks, dv + static_cast<uint64_t>(ks * (2048 >> 4)), kIdO, (i > 0 || ks > 0) ? 1u : 0u);
        if (i == nsteps - 1) tc_commit(bar_o + t * 8);
      };
      if (wait1(bar_q, 0) && wait1(bar_k, 0)) {
        if (lane == 0) {
          for (int t = 0; t < nt; ++t) issue_s(t, 0);
          tc_commit(bar_kf);
        }
        for (int i = 0; i < nsteps && ok_p; ++i) {
          for (int t = 0; t < nt && ok_p; ++t) {
            if (!wait1(bar_p + t * 8, static_cast<uint32_t>(i & 1))) break;
            if (t == 0 && !wait1(bar_v + (i & 1) * 8, static_cast<uint32_t>((i >> 1) & 1))) break;
            if (lane == 0) {
              issue_pv(t, i);
              if (t == nt - 1) tc_commit(bar_vf + (i & 1) * 8);
            }
            if (i + 1 < nsteps) {
              if (t == 0 && !wait1(bar_k + ((i + 1) & 1) * 8, static_cast<uint32_t>(((i + 1) >> 1) & 1))) break;
              if (lane == 0) {
                issue_s(t, i + 1);
                if (t == nt - 1) tc_commit(bar_kf + ((i + 1) & 1) * 8);
              }
            }
            __syncwarp();
          }
        }
      }
      if (lane == 0) {
        if (!ok_p) atomicOr(err, kErrWaitTimeout);
        // every MMA issued above completes before the CTA leaves
        tc_commit(bar_done);
        lane_wait(bar_done, 0, kDrainNs);
      }
    } else {
      // ---- K or V tiles of each step; LWK (LWV) warps per tile ----
      const int lw = warp - C::SOFT / 32 - 1;  // 0 .. LWK + LWV - 1
      const bool vt = lw >= C::LWK;
      const int nlw = vt ? C::LWV : C::LWK;
      const int nb = C::BPS / nlw;  // blocks this warp loads
      const int ib0 = (vt ? lw - C::LWK : lw) * nb;
      const int* trow = p.tables + s * p.t_s;
      const uint64_t policy = l2_policy_evict_normal();
      const uint32_t full = vt ? bar_v : bar_k;
      const uint32_t freed = vt ? bar_vf : bar_kf;
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
        if (j >= 2 && !wait1(freed + (j & 1) * 8, static_cast<uint32_t>(((j - 2) >> 1) & 1))) break;
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
    // ================= softmax warps: one row per thread =================
    const int t = warp >> 2;                 // tile
    const int rl = (warp & 3) * 32 + lane;   // row in the tile = tensor-memory lane
    const int row = r0 + t * 128 + rl;
    const bool row_ok = row < rows_all;
    const int pos = row_ok ? L - n + row / p.g : lim_max;  // padding rows: the CTA's last
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + t * 256 + lane_off, tO = tS + 128;
    // Q row into shared memory (K-major, 128-byte swizzle)
    {
      const uint4* qp = reinterpret_cast<const uint4*>(
          static_cast<const uint16_t*>(p.q) + (q0 + (row_ok ? row / p.g : 0)) * p.q_t +
          (static_cast<long long>(h) * p.g + (row_ok ? row % p.g : 0)) * p.q_h);
      const uint32_t sq = sQ + t * C::TILE;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 v = row_ok ? __ldg(qp + c) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t a = sq + (c >> 3) * C::HALF + (rl >> 3) * 1024 + (rl & 7) * 128 + (((c & 7) ^ (rl & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                     "r"(v.w)
                     : "memory");
      }
      fence_async_smem();  // Q written by the threads, read by the tensor cores
      mbar_arrive(bar_q);
    }
    if (t < nt) {
      const float sl = p.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok_s = true;
      for (int i = 0; i < nsteps; ++i) {
        const int key0 = i * C::KEYS;
        // S_t(i) complete: also O_t += P_t(i - 1) V is (issued before it)
        if (!warp_wait(bar_s + t * 8, static_cast<uint32_t>(i & 1), kWaitNs)) {
          ok_s = false;
          break;
        }
        tc_fence_after();
        // the row's 128 scores, raw (the scale is applied inside the
        // exponent; it is positive); keys past the row's position -inf
        uint32_t v[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, v[c]);
        tmem_wait_ld();
        if (__any_sync(0xffffffffu, key0 + 127 > pos)) {  // masked in place (bits of -inf)
#pragma unroll
          for (int u = 0; u < 128; ++u)
            if (key0 + u > pos) v[u >> 5][u & 31] = 0xff800000u;
        }
        auto x = [&](int u) { return __uint_as_float(v[u >> 5][u & 31]); };
        float mm[4];  // independent chains of 32
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          mm[c] = x(32 * c);
#pragma unroll
          for (int u = 1; u < 31; u += 2) mm[c] = fmax3(mm[c], x(32 * c + u), x(32 * c + u + 1));
          mm[c] = fmaxf(mm[c], x(32 * c + 31));
        }
        const float mx = fmaxf(fmax3(mm[0], mm[1], mm[2]), mm[3]) * sl;
        // The exponent base moves only when the row's max grows by more than
        // 8 (P then stays below 2^8, exact enough in 16 bits and far from
        // fp32 overflow in O and l); otherwise O needs no rescale this step.
        const float m_new = fmaxf(m_run, mx);
        const bool grow = m_new > m_run + 8.f || m_run == -INFINITY;
        const float m_use = grow ? m_new : m_run;
        const float base = m_use == -INFINITY ? 0.f : m_use;
        const float alpha = grow ? exp2f(m_run - base) : 1.f;
        // V rows at or past the sequence's length may hold anything (a
        // partly filled last block): tile A zeroes them (their P is 0 but
        // 0 * NaN is not); both products of the step are issued after P_A
        if (t == 0 && key0 + C::KEYS > L) {
          if (!warp_wait(bar_v + (i & 1) * 8, static_cast<uint32_t>((i >> 1) & 1), kWaitNs)) {
            ok_s = false;
            break;
          }
          const uint32_t dv = sbase + C::OFF_V + (i & 1) * C::TILE;
          for (int k = max(L - key0, 0) * 16 + rl; k < C::KEYS * 16; k += 128) {
            const int key = k >> 4, c = k & 15;  // 16-byte chunk c of key row `key`
            const uint32_t a = dv + (c >> 3) * C::HALF + (key >> 3) * 1024 + (key & 7) * 128 + ((c & 7) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
          }
          fence_async_smem();
        }
        // P = 2^(x sl - base), 16-bit pairs, over the first 64 columns of S
        const uint64_t sl2 = f2_pack(sl, sl), nb2 = f2_pack(-base, -base);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};  // partial row sums, pairs
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            float t0, t1;
            f2_unpack(f2_fma(f2_pack(x(32 * c + u), x(32 * c + u + 1)), sl2, nb2), t0, t1);
            const float p0 = ex2_fast(t0), p1 = ex2_fast(t1);
            acc[(u >> 1) & 3] = f2_add(acc[(u >> 1) & 3], f2_pack(p0, p1));
            pk[u >> 1] = pack2<QBF>(p0, p1);
          }
          tmem_st16(tS + 16 * c, pk);
        }
        // O rescaled after P, when the scores' registers are free again (the
        // product that adds P V is issued only after this thread's arrival)
        if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {  // warp-collective loads / stores
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[16];
            tmem_ld16(tO + 16 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 16; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
            tmem_st16(tO + 16 * c, o);
          }
        }
        float lsum0, lsum1;
        f2_unpack(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), lsum0, lsum1);
        l_run = l_run * alpha + (lsum0 + lsum1);
        m_run = m_use;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p + t * 8);
      }
      if (ok_s && !warp_wait(bar_o + t * 8, 0u, kWaitNs)) ok_s = false;
      if (ok_s) {
        // epilogue: O row / l, 16-bit, to the output row
        tc_fence_after();
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        uint4* orow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) +
                                               (q0 + (row_ok ? row / p.g : 0)) * p.o_t +
                                               (static_cast<long long>(h) * p.g + (row_ok ? row % p.g : 0)) * p.o_h);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 w;
              w.x = pack2<QBF>(__uint_as_float(o[8 * u + 0]) * inv, __uint_as_float(o[8 * u + 1]) * inv);
              w.y = pack2<QBF>(__uint_as_float(o[8 * u + 2]) * inv, __uint_as_float(o[8 * u + 3]) * inv);
              w.z = pack2<QBF>(__uint_as_float(o[8 * u + 4]) * inv, __uint_as_float(o[8 * u + 5]) * inv);
              w.w = pack2<QBF>(__uint_as_float(o[8 * u + 6]) * inv, __uint_as_float(o[8 * u + 7]) * inv);
              orow[4 * c + u] = w;
            }
          }
        }
      } else if (lane == 0) {
        atomicOr(err, kErrWaitTimeout);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}

}  // namespace pkv
