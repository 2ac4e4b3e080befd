// Prefix-aware ("cascade") paged decode for sm_100a.
//
// Requests that share a system prompt point their block tables at the same
// physical blocks ("PagedAttention: treat the cache like virtual memory" and
// "Shared System Prompts & Prefix Caching"). The plain decode reads such a
// block once per request; here it is read once per group: the query heads of
// all members of a group become the N dimension of the prefix products, so
// one K/V tile in shared memory serves every member.
//
// The result is the one paged_attn_decode defines: softmax over all tokens of
// a sequence splits into the shared-prefix tokens and the rest, each side is
// reduced to (running max m, sum l, unnormalised O) and the two are combined
// with the log-sum-exp rule, the same way split-KV pieces are.
//
// Three steps, chained on one stream:
//   1. decode_kernel over the tokens after the prefix (its table rows start
//      skip[s] entries in); a sequence with a prefix leaves (m, l, O) per
//      query head instead of an output row (decode_merge_kernel likewise).
//   2. cascade_prefix_kernel: one CTA per (group, kv head, column chunk of 64
//      query columns, chunk of prefix blocks). A column is one query head of
//      one member (member-major). The CTA's 4 warps take 16 columns each; a
//      ring of NS stages holds one prefix block's K and V tiles (TMA,
//      128-byte swizzle) and every warp reads every stage. Per 16-token tile:
//      S^T = K Q^T with two 8-column n-tiles per warp, online softmax per
//      column, O^T += V^T P^T; partials (m, l, O) per column per chunk.
//   3. cascade_merge_kernel: one warp per (member, query head) folds the
//      prefix chunks' partials and the step-1 partial, normalises and writes
//      the output row.
// With an fp8-e4m3 cache the prefix pass widens the codes to f16 in
// registers as the decode does (q rounded to f16, a bf16 row past the f16
// range scaled by a power of two that its logit scale takes back; the K
// scale folded into the logit scale, the V scale into the partials).
#pragma once

#include "decode.cuh"

namespace pkv {

constexpr int kCasCols = 64;  // query columns per prefix CTA (4 warps x 16)
constexpr int kCasMaxChunk = 256;  // prefix blocks per chunk, at most

// Single-thread bounded wait on an mbarrier phase; false after `limit_ns`.
__device__ __forceinline__ bool lane_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (it == 0) t0 = global_ns();
    else if ((it & 63) == 0 && global_ns() - t0 > limit_ns) return false;
  }
}

struct CascadeParams {
  CUtensorMap tmk;  // K pool viewed as {D, B, Hk, NB}
  CUtensorMap tmv;
  const void* q;
  long long q_s, q_h;
  void* out;
  long long o_s, o_h;
  const int* tables;
  long long t_s;
  const int* prefix_blocks;  // [S]
  const int* group_start;    // [G + 1]
  const int* members;        // [M]
  float scale_log2;
  int S, Hk, g, NB, MB, G, M;
  int ncc;  // column chunks per (group, kv head)
  int nkc;  // prefix-block chunks per column chunk
  int cb;   // prefix blocks per chunk
  int* err;
  float* pre_o;         // [G * Hk * ncc * nkc][kCasCols][D]
  float* pre_ml;        // [G * Hk * ncc * nkc][kCasCols][2]
  const float* suf_o;   // [S * Hq][D] step-1 partials
  const float* suf_ml;  // [S * Hq][2]
  const float* k_scale;  // [Hk], fp8 caches only
  const float* v_scale;
};

template <bool QBF, int D, int BS, int NS, bool FP8 = false>
struct PrefixCfg {
  static constexpr int EB = FP8 ? 1 : 2;     // cache element bytes
  static constexpr int EPR = 128 / EB;       // elements per 128-byte row
  static constexpr int NH = (D * EB) / 128;  // 128-byte column groups per token row
  static constexpr int TILE = BS * D * EB;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int KS = D / 16;
  static constexpr int MT = D / 16;
  static constexpr int TT = BS / 16;
  static constexpr int SMEM = 1024 + NS * STAGE + 2 * NS * 8 + kCasMaxChunk * 4;
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  static_assert(BS % 16 == 0, "block_size must be a multiple of 16");
  static_assert(!FP8 || D == 128, "fp8 caches: head_dim 128");
};

template <bool QBF, int D, int BS, int NS, bool FP8 = false>
__global__ void __launch_bounds__(128, 1) cascade_prefix_kernel(const __grid_constant__ CascadeParams p) {
  using C = PrefixCfg<QBF, D, BS, NS, FP8>;
  constexpr uint64_t kWaitNs = 2000000000ull;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t full = sbase + NS * C::STAGE;
  const uint32_t empty = full + NS * 8;
  int* s_phys = reinterpret_cast<int*>(smem_raw + (sbase - smem_addr(smem_raw)) + NS * C::STAGE + 2 * NS * 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, c = lane & 3;
  const int kc = blockIdx.x, cc = blockIdx.y;
  const int gi = blockIdx.z / p.Hk, h = blockIdx.z % p.Hk;

  // This grid is launched once the decode grid has finished (the split-KV
  // merge before it releases its dependents only after its own wait), so
  // the inputs read here are final; it reads nothing the merge writes.
  // griddepcontrol.wait runs at exit, so that this grid finishing implies the
  // merge finished (the prefix merge after it reads the merge's partials).
  pdl_launch_dependents();
  struct WaitAtExit {
    __device__ ~WaitAtExit() { pdl_wait(); }
  } wait_at_exit;
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i * 8, 1);
      mbar_init(empty + i * 8, 4);
    }
    tma_prefetch_desc(&p.tmk);
    tma_prefetch_desc(&p.tmv);
  }
  fence_mbar_init();

  const int m0 = __ldg(p.group_start + gi), m1 = __ldg(p.group_start + gi + 1);
  if (m0 < 0 || m1 < m0 || m1 > p.M) {
    if (tid == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int first = __ldg(p.members + m0);
  if (first < 0 || first >= p.S) {
    if (tid == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int nb = __ldg(p.prefix_blocks + first);
  if (nb < 0 || nb > p.MB || p.cb > kCasMaxChunk) {
    if (tid == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int ncol = (m1 - m0) * p.g;
  const int b_lo = kc * p.cb, b_hi = min(nb, b_lo + p.cb);
  if (cc * kCasCols >= ncol || b_lo >= b_hi) return;  // nothing of this group here
  const int n = b_hi - b_lo;
  for (int j = tid; j < n; j += 128) {  // the chunk's physical blocks, checked
    int phys = __ldg(p.tables + first * p.t_s + b_lo + j);
    if (phys < 0 || phys >= p.NB) {
      atomicOr(p.err, kErrBadBlock);
      phys = 0;
    }
    s_phys[j] = phys;
  }
  __syncthreads();

  const uint64_t policy = l2_policy_evict_first();
  auto issue = [&](int j) {  // thread 0: prefix block b_lo + j into stage j % NS
    const int stage = j % NS;
    const int phys = s_phys[j];
    const uint32_t bar = full + stage * 8;
    const uint32_t dk = sbase + stage * C::STAGE, dv = dk + C::TILE;
    mbar_arrive_expect_tx(bar, C::STAGE);
#pragma unroll
    for (int hh = 0; hh < C::NH; ++hh)
      tma_load_4d(dk + hh * BS * 128, &p.tmk, bar, hh * C::EPR, 0, h, phys, policy);
#pragma unroll
    for (int hh = 0; hh < C::NH; ++hh)
      tma_load_4d(dv + hh * BS * 128, &p.tmv, bar, hh * C::EPR, 0, h, phys, policy);
  };
  if (tid == 0)
    for (int j = 0; j < min(NS, n); ++j) issue(j);

  // Q^T fragments of this warp's 16 columns: n-tile jt holds columns
  // cc * 64 + warp * 16 + jt * 8 + (0..7); lane r carries column 8 jt + r.
  // fp8: the k-slot order of the widened tile puts dims 4c, 4c + 1 in slots
  // 2c, 2c + 1 and dims 4c + 2, 4c + 3 in slots 2c + 8, 2c + 9 of each
  // 16-dim step; q is rounded to f16 (a bf16 row of 2^16 and up first
  // scaled by 2^-e) and slj holds the logit scales of this lane's two
  // accumulator columns (K scale and 2^e included).
  uint32_t qb[2][C::KS][2];
  bool col_ok[2][2];
  float slj[2][2];
  const float sl_base = FP8 ? p.scale_log2 * __ldg(p.k_scale + h) : p.scale_log2;
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
    const int col = cc * kCasCols + warp * 16 + jt * 8 + r;
    const bool ok = col < ncol;
    const int mi = ok ? col / p.g : 0;
    const int s = ok ? __ldg(p.members + m0 + mi) : 0;
    const bool s_ok = ok && s >= 0 && s < p.S;
    const long long qoff = s * p.q_s + (static_cast<long long>(h) * p.g + col % p.g) * p.q_h;
    slj[jt][0] = slj[jt][1] = sl_base;
    if constexpr (!FP8) {
      const uint32_t* qp = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.q) + qoff);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        qb[jt][ks][0] = s_ok ? __ldg(qp + (ks * 16 + 2 * c) / 2) : 0u;
        qb[jt][ks][1] = s_ok ? __ldg(qp + (ks * 16 + 8 + 2 * c) / 2) : 0u;
      }
    } else {
      const uint2* qp = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.q) + qoff);
      float f[C::KS][4];
      float amax = 0.f;
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        const uint2 v = s_ok ? __ldg(qp + (ks * 16 + 4 * c) / 4) : make_uint2(0u, 0u);
        if constexpr (QBF) {
          f[ks][0] = __uint_as_float(v.x << 16);
          f[ks][1] = __uint_as_float(v.x & 0xffff0000u);
          f[ks][2] = __uint_as_float(v.y << 16);
          f[ks][3] = __uint_as_float(v.y & 0xffff0000u);
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f[ks][0]), fabsf(f[ks][1])),
                                   fmaxf(fabsf(f[ks][2]), fabsf(f[ks][3]))));
        } else {
          const __half2 a2 = *reinterpret_cast<const __half2*>(&v.x);
          const __half2 b2 = *reinterpret_cast<const __half2*>(&v.y);
          f[ks][0] = __low2float(a2);
          f[ks][1] = __high2float(a2);
          f[ks][2] = __low2float(b2);
          f[ks][3] = __high2float(b2);
        }
      }
      float qs = 1.f;
      if constexpr (QBF) {  // the row of column 8 jt + r is held by lanes 4r .. 4r + 3
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int ex = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu) - 127;
        const int e = ex >= 16 ? ex - 15 : 0;
        qs = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
        const int e0 = __shfl_sync(0xffffffffu, e, 8 * c), e1 = __shfl_sync(0xffffffffu, e, 8 * c + 4);
        slj[jt][0] = sl_base * __uint_as_float(static_cast<uint32_t>(127 + e0) << 23);
        slj[jt][1] = sl_base * __uint_as_float(static_cast<uint32_t>(127 + e1) << 23);
      }
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        qb[jt][ks][0] = pack2<false>(f[ks][0] * qs, f[ks][1] * qs);
        qb[jt][ks][1] = pack2<false>(f[ks][2] * qs, f[ks][3] * qs);
      }
    }
    // the two accumulator columns of this lane: 8 jt + 2c and + 1
    const int cb0 = cc * kCasCols + warp * 16 + jt * 8 + 2 * c;
    col_ok[jt][0] = cb0 < ncol;
    col_ok[jt][1] = cb0 + 1 < ncol;
  }

  float acc[2][C::MT][4];
  float mrun[2][2], lrun[2][2];
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) acc[jt][mt][0] = acc[jt][mt][1] = acc[jt][mt][2] = acc[jt][mt][3] = 0.f;
    mrun[jt][0] = mrun[jt][1] = -INFINITY;
    lrun[jt][0] = lrun[jt][1] = 0.f;
  }
  bool failed = false;
  int issued = min(NS, n);  // thread 0's count of blocks issued
  int jfail = n;            // first block this warp gave up on

  for (int j = 0; j < n; ++j) {
    const int stage = j % NS;
    const uint32_t parity = static_cast<uint32_t>((j / NS) & 1);
    if (!warp_wait(full + stage * 8, parity, kWaitNs)) {
      if (lane == 0) atomicOr(p.err, kErrWaitTimeout);
      failed = true;
      jfail = j;
      break;
    }
    const uint32_t tk = sbase + stage * C::STAGE, tv = tk + C::TILE;
#pragma unroll
    for (int tt = 0; tt < C::TT; ++tt) {
      // S^T = K Q^T for both n-tiles (K fragments shared)
      float sacc[2][4];
#pragma unroll
      for (int jt = 0; jt < 2; ++jt) sacc[jt][0] = sacc[jt][1] = sacc[jt][2] = sacc[jt][3] = 0.f;
      const int trow = tt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      if constexpr (!FP8) {
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(tk + swz<BS>(trow, ks * 32 + (lane >> 4) * 16), a0, a1, a2, a3);
#pragma unroll
          for (int jt = 0; jt < 2; ++jt) mma16816<QBF>(sacc[jt], a0, a1, a2, a3, qb[jt][ks][0], qb[jt][ks][1]);
        }
      } else {
#pragma unroll
        for (int kp = 0; kp < C::KS / 2; ++kp) {
          uint32_t x0, x1, x2, x3;
          ldsm_x4(tk + swz<BS>(trow, kp * 32 + (lane >> 4) * 16), x0, x1, x2, x3);
          uint32_t a0, a2, a1, a3, b0, b2, b1, b3;
          e4m3x4_to_f16x2x2(x0, a0, a2);
          e4m3x4_to_f16x2x2(x1, a1, a3);
          e4m3x4_to_f16x2x2(x2, b0, b2);
          e4m3x4_to_f16x2x2(x3, b1, b3);
#pragma unroll
          for (int jt = 0; jt < 2; ++jt) {
            mma16816<false>(sacc[jt], a0, a1, a2, a3, qb[jt][2 * kp][0], qb[jt][2 * kp][1]);
            mma16816<false>(sacc[jt], b0, b1, b2, b3, qb[jt][2 * kp + 1][0], qb[jt][2 * kp + 1][1]);
          }
        }
      }
      // online softmax per column (every prefix token is valid)
      uint32_t pb[2][2];
#pragma unroll
      for (int jt = 0; jt < 2; ++jt) {
        const float x0 = sacc[jt][0] * slj[jt][0], x1 = sacc[jt][1] * slj[jt][1];
        const float x2 = sacc[jt][2] * slj[jt][0], x3 = sacc[jt][3] * slj[jt][1];
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = fmaxf(mrun[jt][0], mx0), mn1 = fmaxf(mrun[jt][1], mx1);
        const float al0 = ex2_fast(mrun[jt][0] - mn0), al1 = ex2_fast(mrun[jt][1] - mn1);
        lrun[jt][0] *= al0;
        lrun[jt][1] *= al1;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          acc[jt][mt][0] *= al0;
          acc[jt][mt][1] *= al1;
          acc[jt][mt][2] *= al0;
          acc[jt][mt][3] *= al1;
        }
        mrun[jt][0] = mn0;
        mrun[jt][1] = mn1;
        const float p0 = ex2_fast(x0 - mn0), p1 = ex2_fast(x1 - mn1);
        const float p2 = ex2_fast(x2 - mn0), p3 = ex2_fast(x3 - mn1);
        lrun[jt][0] += p0 + p2;
        lrun[jt][1] += p1 + p3;
        pb[jt][0] = movmatrix_t(pack2<QBF && !FP8>(p0, p1));
        pb[jt][1] = movmatrix_t(pack2<QBF && !FP8>(p2, p3));
      }
      // O^T += V^T P^T (V fragments shared by both n-tiles; fp8: one
      // transposed load covers two m-tiles, widened to f16)
      if constexpr (!FP8) {
#pragma unroll
        for (int i = 0; i < C::MT; ++i) {
          const int vrow = tt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
          uint32_t f0, f1, f2, f3;
          ldsm_x4_t(tv + swz<BS>(vrow, i * 32 + ((lane >> 3) & 1) * 16), f0, f1, f2, f3);
#pragma unroll
          for (int jt = 0; jt < 2; ++jt) mma16816<QBF>(acc[jt][i], f0, f1, f2, f3, pb[jt][0], pb[jt][1]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < C::MT / 2; ++i) {
          const int vrow = tt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          uint32_t x0, x1, x2, x3, f[8];
          ldsm_x4_t(tv + swz<BS>(vrow, i * 32 + (lane >> 4) * 16), x0, x1, x2, x3);
          // bytes (d, t), (d + 1, t), (d, t + 1), (d + 1, t + 1) -> token
          // pairs (d, t | t + 1) and (d + 1, t | t + 1)
          e4m3x4_to_f16x2x2(prmt(x0, 0, 0x3120), f[0], f[1]);
          e4m3x4_to_f16x2x2(prmt(x1, 0, 0x3120), f[2], f[3]);
          e4m3x4_to_f16x2x2(prmt(x2, 0, 0x3120), f[4], f[5]);
          e4m3x4_to_f16x2x2(prmt(x3, 0, 0x3120), f[6], f[7]);
#pragma unroll
          for (int jt = 0; jt < 2; ++jt) {
            mma16816<false>(acc[jt][2 * i], f[0], f[1], f[2], f[3], pb[jt][0], pb[jt][1]);
            mma16816<false>(acc[jt][2 * i + 1], f[4], f[5], f[6], f[7], pb[jt][0], pb[jt][1]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + stage * 8);
    if (tid == 0 && j + NS < n) {
      // the stage is refilled once all four warps have read it
      if (!lane_wait(empty + stage * 8, parity, kWaitNs)) {
        atomicOr(p.err, kErrWaitTimeout);
      } else {
        issue(j + NS);
        ++issued;
      }
    }
  }
  if (failed) {
    // let copies still in flight (issued, not yet waited for) land before the
    // CTA's shared memory is reused
    if (tid == 0)
      for (int i = jfail; i < issued; ++i)
        lane_wait(full + (i % NS) * 8, static_cast<uint32_t>((i / NS) & 1), 100000000ull);
    return;
  }

  // partials of this chunk: one row of D floats (and m, l) per column, O
  // scaled by the V scale (fp8)
  const float vs = FP8 ? __ldg(p.v_scale + h) : 1.f;
  const long long item = ((static_cast<long long>(blockIdx.z) * p.ncc + cc) * p.nkc + kc);
  float* po = p.pre_o + item * kCasCols * D;
  float* pm = p.pre_ml + item * kCasCols * 2;
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
    float l0 = lrun[jt][0], l1 = lrun[jt][1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    const int cl = warp * 16 + jt * 8 + 2 * c;  // column within the chunk
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt) {
      const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
      const int db = FP8 ? da + 1 : da + 8;
      if (col_ok[jt][0]) {
        po[cl * D + da] = acc[jt][mt][0] * vs;
        po[cl * D + db] = acc[jt][mt][2] * vs;
      }
      if (col_ok[jt][1]) {
        po[(cl + 1) * D + da] = acc[jt][mt][1] * vs;
        po[(cl + 1) * D + db] = acc[jt][mt][3] * vs;
      }
    }
    if (r == 0) {
      if (col_ok[jt][0]) {
        pm[cl * 2] = mrun[jt][0];
        pm[cl * 2 + 1] = l0;
      }
      if (col_ok[jt][1]) {
        pm[(cl + 1) * 2] = mrun[jt][1];
        pm[(cl + 1) * 2 + 1] = l1;
      }
    }
  }
}

// One warp per (member j, query head hq), grid (members x heads, groups):
// fold the prefix chunks of j's group and the partial of j's own tokens,
// normalise, write out[s, hq].
template <bool QBF, int D>
__global__ void __launch_bounds__(128) cascade_merge_kernel(const __grid_constant__ CascadeParams p) {
  // The group data are inputs of the call: read them before waiting for the
  // prefix grid (and through it the split-KV merge), whose partials follow.
  // Every thread waits before it exits, so this grid finishing implies the
  // kernels before it finished.
  pdl_launch_dependents();
  struct WaitAtExit {
    __device__ ~WaitAtExit() { pdl_wait(); }
  } wait_at_exit;
  const int lane = threadIdx.x & 31;
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int Hq = p.Hk * p.g;
  const int gi = blockIdx.y;
  const int m0 = __ldg(p.group_start + gi), m1 = __ldg(p.group_start + gi + 1);
  if (blockIdx.x == 0 && threadIdx.x == 0 &&
      static_cast<long long>(m1 - m0) * Hq > static_cast<long long>(gridDim.x) * (blockDim.x >> 5))
    atomicOr(p.err, kErrBadLen);  // a group larger than max_group_size
  if (wid >= static_cast<long long>(m1 - m0) * Hq) return;
  const int jl = static_cast<int>(wid / Hq), hq = static_cast<int>(wid % Hq);
  if (m0 < 0 || m1 > p.M) {
    if (lane == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int s = __ldg(p.members + m0 + jl);
  if (s < 0 || s >= p.S) {
    if (lane == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int h = hq / p.g;
  const int col = jl * p.g + hq % p.g;
  const int cc = col / kCasCols, cl = col % kCasCols;
  if (cc >= p.ncc) {  // a group larger than the launch was sized for
    if (lane == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int nb = __ldg(p.prefix_blocks + s);  // equal for all members
  const int nk = min(p.nkc, (max(nb, 0) + p.cb - 1) / p.cb);
  const long long item0 = (static_cast<long long>(gi * p.Hk + h) * p.ncc + cc) * p.nkc;
  const long long srow = static_cast<long long>(s) * Hq + hq;
  pdl_wait();  // (a second wait at exit returns at once)

  // pieces: prefix chunks 0 .. nk-1, then the sequence's own partial (nk).
  // Lane k holds piece base + k's (m, l); all row loads of a batch are in
  // flight together.
  constexpr int V = D / 32;  // floats per lane
  float mx = -INFINITY, lsum = 0.f, a[V];
#pragma unroll
  for (int v = 0; v < V; ++v) a[v] = 0.f;
  for (int base = 0; base <= nk; base += 32) {
    const int k = base + lane;
    float m = -INFINITY, l = 0.f;
    if (k <= nk) {
      const float* ml = k < nk ? p.pre_ml + ((item0 + k) * kCasCols + cl) * 2 : p.suf_ml + srow * 2;
      m = ml[0];
      l = ml[1];
    }
    float cm = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    if (cm == -INFINITY) continue;  // nothing in this batch
    const float mn = fmaxf(mx, cm);
    const float sa = mx == -INFINITY ? 0.f : exp2f(mx - mn);
    lsum *= sa;
#pragma unroll
    for (int v = 0; v < V; ++v) a[v] *= sa;
    mx = mn;
    const float w = m == -INFINITY ? 0.f : exp2f(m - mn);
    float lw = l * w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
    lsum += lw;
    const int cnt = min(32, nk + 1 - base);
    for (int k0 = 0; k0 < cnt; k0 += 8) {
      float x[8][V];
      float wk[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int kk = base + k0 + u;
        wk[u] = __shfl_sync(0xffffffffu, w, (k0 + u) & 31);
        if (k0 + u < cnt && wk[u] != 0.f) {
          const float* o = kk < nk ? p.pre_o + ((item0 + kk) * kCasCols + cl) * D : p.suf_o + srow * D;
#pragma unroll
          for (int v = 0; v < V; ++v) x[u][v] = o[lane * V + v];
        } else {
#pragma unroll
          for (int v = 0; v < V; ++v) x[u][v] = 0.f;
          wk[u] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int v = 0; v < V; ++v) a[v] += x[u][v] * wk[u];
    }
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  uint16_t* oh = static_cast<uint16_t*>(p.out) + s * p.o_s + hq * p.o_h + lane * V;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    if constexpr (QBF) oh[v] = __bfloat16_as_ushort(__float2bfloat16_rn(a[v] * inv));
    else oh[v] = __half_as_ushort(__float2half_rn(a[v] * inv));
  }
}

}  // namespace pkv
