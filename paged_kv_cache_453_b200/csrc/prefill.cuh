// Multi-token (causal) paged attention for sm_100a: several new tokens of a
// sequence attend over its paged cache in one call (a prompt or a chunk of
// it after its K/V went into the blocks allocated for it, "How Block Paging
// Operates During Generation" and "Dynamic Request Insertion"; speculative
// tokens being verified). Sequence s has n_s new tokens, the last n_s of its
// L_s; query row q_start[s] + j is the token at position L_s - n_s + j and
// attends to positions 0 .. L_s - n_s + j through the block table.
//
// One CTA per (sequence, kv head, chunk of NW * 16 query columns), a column
// being one query head of one new token (token-major). NW warps of 16
// columns (two 8-column n-tiles) share a ring of NS stages that holds one
// block's K and V tiles (TMA, 128-byte swizzle; warp 0 issues, every warp
// reads every stage), so each K/V byte crosses HBM once per chunk. Per
// 16-token tile: S^T = K Q^T (K fragments shared by the n-tiles), keys past a
// column's position masked to -inf (blocks wholly before the chunk's first
// position need no mask), online softmax per column in the exp2 domain,
// O^T += V^T P^T with V rows past the sequence zeroed. Each column's output
// row is normalised and written at the end.
//
// Short queries over long, uneven contexts (speculative verification) give
// too few, unequal CTAs; there the blocks of each (sequence, head) are also
// cut into chunks of kv_chunk blocks, one CTA each, which leave fp32
// partials (m, l, unnormalised O) per column, and prefill_merge_kernel folds
// a row's chunks with the log-sum-exp rule.
//
// An fp8-e4m3 cache is read as the decode reads it: codes widened to f16 in
// registers, q rounded to f16 (a bf16 row reaching 2^16 first scaled by a
// power of two that its logit scale takes back), the K scale folded into the
// logit scale and the V scale into the output (or the partials).
#pragma once

#include "cascade.cuh"

namespace pkv {

struct PrefillParams {
  CUtensorMap tmk;  // K pool viewed as {D, B, Hk, NB}
  CUtensorMap tmv;
  const void* q;
  long long q_t, q_h;  // element strides of q [T, Hq, D]
  void* out;
  long long o_t, o_h;
  const int* tables;
  long long t_s;
  const int* lens;
  const int* q_start;  // [S + 1]
  float scale_log2;
  int S, T, Hk, g, NB, MB, BS;
  int evict_first;  // L2 hint for K/V tiles: 1 when one chunk reads them
  int* err;
  int nkv;          // KV chunks per (sequence, head); 1: no split, outputs written directly
  int ccols;        // query columns per CTA (the kernel's NW * 16)
  int kv_chunk;     // blocks per KV chunk (split only)
  float* part_o;    // [T * Hq * nkv][D] (split only)
  float* part_ml;   // [T * Hq * nkv][2]
  const int* order;  // [S] sequences by decreasing context length, or null (tensor-core kernels)
  const float* k_scale;  // [Hk], fp8 caches only
  const float* v_scale;
};

// order[r] = the sequence with the r-th longest context (ties: lower index
// first); one CTA of 1024 threads, S <= 1024 (each thread counts its
// sequence's rank over the lengths staged in shared memory). Its dependents
// may start their prologue at once; they read order only after their
// grid-dependency wait.
constexpr int kOrderMaxSeqs = 1024;
__global__ void __launch_bounds__(kOrderMaxSeqs) order_by_len_kernel(const int* lens, int S, int* order) {
  __shared__ int sl[kOrderMaxSeqs];
  pdl_launch_dependents();
  const int i = threadIdx.x;
  const int li = i < S ? lens[i] : 0;
  sl[i] = li;
  __syncthreads();
  if (i < S) {
    int rank = 0;
    for (int j = 0; j < S; ++j) {
      const int lj = sl[j];
      rank += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    order[rank] = i;
  }
}

template <bool QBF, int D, int BS, int NS, int NW, bool FP8 = false>
struct PrefillCfg {
  static constexpr int EB = FP8 ? 1 : 2;     // cache element bytes
  static constexpr int EPR = 128 / EB;       // elements per 128-byte row
  static constexpr int NH = (D * EB) / 128;  // 128-byte column groups per token row
  static constexpr int TILE = BS * D * EB;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int KS = D / 16;
  static constexpr int MT = D / 16;
  static constexpr int TT = BS / 16;
  static constexpr int COLS = NW * 16;
  static constexpr int SMEM = 1024 + NS * STAGE + 2 * NS * 8;
  static_assert(D % 64 == 0 && BS % 16 == 0, "head_dim multiple of 64, block_size of 16");
  static_assert(!FP8 || D == 128, "fp8 caches: head_dim 128");
};

template <bool QBF, int D, int BS, int NS, int NW, bool FP8 = false>
__global__ void __launch_bounds__(NW * 32, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
  using C = PrefillCfg<QBF, D, BS, NS, NW, FP8>;
  constexpr uint64_t kWaitNs = 2000000000ull;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const uint32_t full = sbase + NS * C::STAGE;
  const uint32_t empty = full + NS * 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane >> 2, c = lane & 3;
  // grid: x = column chunk, y = KV chunk, z = (sequence, head)
  const long long sh = blockIdx.z;
  const int s = static_cast<int>(sh / p.Hk), h = static_cast<int>(sh % p.Hk);
  const int kc = blockIdx.y;

  pdl_launch_dependents();
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i * 8, 1);
      mbar_init(empty + i * 8, NW);
    }
    tma_prefetch_desc(&p.tmk);
    tma_prefetch_desc(&p.tmv);
  }
  fence_mbar_init();
  __syncthreads();
  pdl_wait();
  if (s >= p.S) return;

  const int q0 = __ldg(p.q_start + s), q1 = __ldg(p.q_start + s + 1);
  const int L = __ldg(p.lens + s);
  const int n = q1 - q0;
  if (n < 0 || L < n || L > p.MB * BS || q0 < 0 || q1 > p.T) {
    if (tid == 0 && blockIdx.x == 0) atomicOr(p.err, kErrBadLen);
    return;
  }
  const int cols = n * p.g;
  const int col0 = blockIdx.x * C::COLS;
  if (tid == 0 && blockIdx.x == 0 && kc == 0 && cols > static_cast<int>(gridDim.x) * C::COLS)
    atomicOr(p.err, kErrBadLen);  // more new tokens than max_q_tokens
  if (col0 >= cols) return;
  const int cend = min(cols, col0 + C::COLS);
  const int lim_max = L - n + (cend - 1) / p.g;   // last position any column attends to
  const int lim_min = L - n + col0 / p.g;         // first column's position
  const int nblk_all = lim_max / BS + 1;
  const int plain_blocks = (lim_min + 1) / BS;    // blocks no column needs masked
  const int b_lo = p.nkv > 1 ? kc * p.kv_chunk : 0;
  const int b_hi = p.nkv > 1 ? min(nblk_all, b_lo + p.kv_chunk) : nblk_all;
  if (b_lo >= b_hi) return;                       // no keys of this chunk here
  const int nblk = b_hi - b_lo;                    // blocks b_lo + j, j < nblk

  // warp 0: table entries of blocks 32w .. 32w + 31 (window w) and the next
  int win = b_lo >> 5, tw_cur = 0, tw_nxt = 0;
  const int* trow = p.tables + s * p.t_s;
  if (warp == 0) {
    tw_cur = 32 * win + lane < nblk_all ? __ldg(trow + 32 * win + lane) : 0;
    tw_nxt = 32 * (win + 1) + lane < nblk_all ? __ldg(trow + 32 * (win + 1) + lane) : 0;
  }
  const uint64_t policy = p.evict_first ? l2_policy_evict_first() : l2_policy_evict_normal();
  auto issue = [&](int j) {  // warp 0, all lanes: block b_lo + j into stage j % NS
    const int b = b_lo + j;
    if ((b >> 5) != win) {   // next window: shift, fetch the one after
      win = b >> 5;
      tw_cur = tw_nxt;
      const int nb2 = 32 * (win + 1) + lane;
      tw_nxt = nb2 < nblk_all ? __ldg(trow + nb2) : 0;
    }
    int phys = __shfl_sync(0xffffffffu, tw_cur, b & 31);
    if (phys < 0 || phys >= p.NB) {
      if (lane == 0) atomicOr(p.err, kErrBadBlock);
      phys = 0;
    }
    if (lane == 0) {
      const int stage = j % NS;
      const uint32_t bar = full + stage * 8;
      const uint32_t dk = sbase + stage * C::STAGE, dv = dk + C::TILE;
      mbar_arrive_expect_tx(bar, C::STAGE);
#pragma unroll
      for (int hh = 0; hh < C::NH; ++hh)
        tma_load_4d(dk + hh * BS * 128, &p.tmk, bar, hh * C::EPR, 0, h, phys, policy);
#pragma unroll
      for (int hh = 0; hh < C::NH; ++hh)
        tma_load_4d(dv + hh * BS * 128, &p.tmv, bar, hh * C::EPR, 0, h, phys, policy);
    }
  };
  int issued = 0;
  if (warp == 0) {
    for (; issued < min(NS, nblk); ++issued) issue(issued);
  }

  // Q^T fragments of this warp's columns; lane r carries column 8 jt + r.
  // fp8: the widened tile's k-slots 2c, 2c + 1 hold dims 4c, 4c + 1 and
  // slots 2c + 8, 2c + 9 dims 4c + 2, 4c + 3 of each 16-dim step; slj are
  // the logit scales of this lane's two accumulator columns.
  const bool active = col0 + warp * 16 < cols;
  uint32_t qb[2][C::KS][2];
  int lim[2][2];  // positions of this lane's two accumulator columns per n-tile
  bool col_ok[2][2];
  float slj[2][2];
  const float sl_base = FP8 ? p.scale_log2 * __ldg(p.k_scale + h) : p.scale_log2;
#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
    const int col = col0 + warp * 16 + jt * 8 + r;
    const bool ok = col < cols;
    const int tok = ok ? col / p.g : 0;
    const long long qoff = (q0 + tok) * p.q_t + (static_cast<long long>(h) * p.g + (ok ? col % p.g : 0)) * p.q_h;
    slj[jt][0] = slj[jt][1] = sl_base;
    if constexpr (!FP8) {
      const uint32_t* qp = reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(p.q) + qoff);
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        qb[jt][ks][0] = ok ? __ldg(qp + (ks * 16 + 2 * c) / 2) : 0u;
        qb[jt][ks][1] = ok ? __ldg(qp + (ks * 16 + 8 + 2 * c) / 2) : 0u;
      }
    } else {
      const uint2* qp = reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.q) + qoff);
      float f[C::KS][4];
      float amax = 0.f;
#pragma unroll
      for (int ks = 0; ks < C::KS; ++ks) {
        const uint2 v = ok ? __ldg(qp + (ks * 16 + 4 * c) / 4) : make_uint2(0u, 0u);
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
    const int cb0 = col0 + warp * 16 + jt * 8 + 2 * c;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      col_ok[jt][u] = cb0 + u < cols;
      // a column past the end attends like the last one (finite, not written)
      lim[jt][u] = col_ok[jt][u] ? L - n + (cb0 + u) / p.g : lim_max;
    }
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
  int jfail = nblk;

  for (int j = 0; j < nblk; ++j) {
    const int b = b_lo + j;
    const int stage = j % NS;
    const uint32_t parity = static_cast<uint32_t>((j / NS) & 1);
    if (!warp_wait(full + stage * 8, parity, kWaitNs)) {
      if (lane == 0) atomicOr(p.err, kErrWaitTimeout);
      jfail = j;
      break;
    }
    if (active) {
      const uint32_t tk = sbase + stage * C::STAGE, tv = tk + C::TILE;
      const bool masked = b >= plain_blocks;
      const int nvalid = min(BS, L - b * BS);  // rows holding tokens
#pragma unroll
      for (int tt = 0; tt < C::TT; ++tt) {
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
        const int k0 = b * BS + tt * 16 + r, k1 = k0 + 8;  // keys of this lane's rows
        uint32_t pb[2][2];
#pragma unroll
        for (int jt = 0; jt < 2; ++jt) {
          // a lane's two columns as packed f32x2 pairs
          const uint64_t sl2 = f2_pack(slj[jt][0], slj[jt][1]);
          float x0, x1, x2, x3;
          f2_unpack(f2_mul(f2_pack(sacc[jt][0], sacc[jt][1]), sl2), x0, x1);
          f2_unpack(f2_mul(f2_pack(sacc[jt][2], sacc[jt][3]), sl2), x2, x3);
          if (masked) {
            x0 = k0 <= lim[jt][0] ? x0 : -INFINITY;
            x1 = k0 <= lim[jt][1] ? x1 : -INFINITY;
            x2 = k1 <= lim[jt][0] ? x2 : -INFINITY;
            x3 = k1 <= lim[jt][1] ? x3 : -INFINITY;
          }
          float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
          // The exponent base moves only when a score passes it by more than
          // 8 (P stays at or below 2^8, rounded to 16 bits with the same
          // relative error): until then neither the column maxima across the
          // warp nor a rescale of O is needed. When it moves it becomes the
          // column's running maximum. A column with no key yet (every key so
          // far past its position, only in a later KV chunk) keeps m = -inf,
          // l = 0, O = 0, and its exponent base is 0 instead of -inf.
          if (__any_sync(0xffffffffu, mx0 > mrun[jt][0] + 8.f || mx1 > mrun[jt][1] + 8.f)) {
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
              mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
              mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
            }
            const float mn0 = fmaxf(mrun[jt][0], mx0), mn1 = fmaxf(mrun[jt][1], mx1);
            const float n0 = mn0 == -INFINITY ? 0.f : mn0, n1 = mn1 == -INFINITY ? 0.f : mn1;
            const float al0 = ex2_fast(mrun[jt][0] - n0), al1 = ex2_fast(mrun[jt][1] - n1);
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
          }
          const uint64_t nb2 = f2_pack(mrun[jt][0] == -INFINITY ? 0.f : -mrun[jt][0],
                                       mrun[jt][1] == -INFINITY ? 0.f : -mrun[jt][1]);
          float a0, a1, a2, a3;
          f2_unpack(f2_add(f2_pack(x0, x1), nb2), a0, a1);
          f2_unpack(f2_add(f2_pack(x2, x3), nb2), a2, a3);
          const float p0 = ex2_fast(a0), p1 = ex2_fast(a1);
          const float p2 = ex2_fast(a2), p3 = ex2_fast(a3);
          f2_unpack(f2_add(f2_pack(lrun[jt][0], lrun[jt][1]), f2_add(f2_pack(p0, p1), f2_pack(p2, p3))),
                    lrun[jt][0], lrun[jt][1]);
          pb[jt][0] = movmatrix_t(pack2<QBF && !FP8>(p0, p1));
          pb[jt][1] = movmatrix_t(pack2<QBF && !FP8>(p2, p3));
        }
        // V rows past the sequence's tokens zeroed (their P is 0, a NaN
        // there would still poison the sum)
        const int tb = tt * 16 + 2 * c;
        const uint32_t keep01 = (tb < nvalid ? 0x0000ffffu : 0u) | (tb + 1 < nvalid ? 0xffff0000u : 0u);
        const uint32_t keep23 = (tb + 8 < nvalid ? 0x0000ffffu : 0u) | (tb + 9 < nvalid ? 0xffff0000u : 0u);
        if constexpr (!FP8) {
#pragma unroll
          for (int i = 0; i < C::MT; ++i) {
            const int vrow = tt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            uint32_t f0, f1, f2, f3;
            ldsm_x4_t(tv + swz<BS>(vrow, i * 32 + ((lane >> 3) & 1) * 16), f0, f1, f2, f3);
            f0 &= keep01;
            f1 &= keep01;
            f2 &= keep23;
            f3 &= keep23;
#pragma unroll
            for (int jt = 0; jt < 2; ++jt) mma16816<QBF>(acc[jt][i], f0, f1, f2, f3, pb[jt][0], pb[jt][1]);
          }
        } else {  // one transposed load covers two m-tiles, widened to f16
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
            f[0] &= keep01;
            f[1] &= keep01;
            f[2] &= keep23;
            f[3] &= keep23;
            f[4] &= keep01;
            f[5] &= keep01;
            f[6] &= keep23;
            f[7] &= keep23;
#pragma unroll
            for (int jt = 0; jt < 2; ++jt) {
              mma16816<false>(acc[jt][2 * i], f[0], f[1], f[2], f[3], pb[jt][0], pb[jt][1]);
              mma16816<false>(acc[jt][2 * i + 1], f[4], f[5], f[6], f[7], pb[jt][0], pb[jt][1]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + stage * 8);
    if (warp == 0 && j + NS < nblk) {
      // refill once every warp has read the stage
      bool ok = true;
      if (lane == 0) ok = lane_wait(empty + stage * 8, parity, kWaitNs);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) atomicOr(p.err, kErrWaitTimeout);
      } else {
        issue(j + NS);
        ++issued;
      }
    }
  }
  if (jfail < nblk) {
    // copies still in flight (issued, not waited for) land before the CTA's
    // shared memory is reused
    if (warp == 0 && lane == 0)
      for (int i = jfail; i < issued; ++i)
        lane_wait(full + (i % NS) * 8, static_cast<uint32_t>((i / NS) & 1), 100000000ull);
    return;
  }
  if (!active) return;

#pragma unroll
  for (int jt = 0; jt < 2; ++jt) {
    float l0 = lrun[jt][0], l1 = lrun[jt][1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    const float vs = FP8 ? __ldg(p.v_scale + h) : 1.f;  // O carries the V scale
    const float i0 = l0 > 0.f ? vs / l0 : 0.f, i1 = l1 > 0.f ? vs / l1 : 0.f;
    const int cb0 = col0 + warp * 16 + jt * 8 + 2 * c;
    if (p.nkv > 1) {  // partials of this KV chunk
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (!col_ok[jt][u]) continue;
        const int col = cb0 + u;
        const long long row = (static_cast<long long>(q0 + col / p.g) * (p.Hk * p.g) +
                               static_cast<long long>(h) * p.g + col % p.g) * p.nkv + kc;
        float* po = p.part_o + row * D;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
          const int db = FP8 ? da + 1 : da + 8;
          po[da] = acc[jt][mt][u] * vs;
          po[db] = acc[jt][mt][u + 2] * vs;
        }
        if (r == 0) {
          p.part_ml[row * 2] = mrun[jt][u];
          p.part_ml[row * 2 + 1] = u ? l1 : l0;
        }
      }
      continue;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (!col_ok[jt][u]) continue;
      const int col = cb0 + u;
      uint16_t* o = static_cast<uint16_t*>(p.out) + (q0 + col / p.g) * p.o_t +
                    (static_cast<long long>(h) * p.g + col % p.g) * p.o_h;
      const float inv = u ? i1 : i0;
#pragma unroll
      for (int mt = 0; mt < C::MT; ++mt) {
        const float x = acc[jt][mt][u] * inv, y = acc[jt][mt][u + 2] * inv;
        const int da = FP8 ? 16 * mt + 2 * r : 16 * mt + r;
        const int db = FP8 ? da + 1 : da + 8;
        if constexpr (QBF) {
          o[da] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
          o[db] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
        } else {
          o[da] = __half_as_ushort(__float2half_rn(x));
          o[db] = __half_as_ushort(__float2half_rn(y));
        }
      }
    }
  }
}

// One warp per (new token row, query head), grid (rows x heads of a
// sequence, sequences): fold the row's KV-chunk partials (chunks whose keys
// all lie past the row's position hold m = -inf and are skipped) and write
// the normalised output.
template <bool QBF, int D>
__global__ void __launch_bounds__(128) prefill_merge_kernel(const __grid_constant__ PrefillParams p) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int s = blockIdx.y;
  const int Hq = p.Hk * p.g;
  const int q0 = __ldg(p.q_start + s), q1 = __ldg(p.q_start + s + 1);
  const int L = __ldg(p.lens + s);
  const int n = q1 - q0;
  if (n < 0 || L < n || L > p.MB * p.BS || q0 < 0 || q1 > p.T) return;  // flagged by the kernel
  if (wid >= static_cast<long long>(n) * Hq) return;
  const int j = static_cast<int>(wid / Hq), hq = static_cast<int>(wid % Hq);
  const long long row = (static_cast<long long>(q0 + j) * Hq + hq) * p.nkv;
  // chunks written for this row: those with keys before the last position of
  // its column chunk (the kernel's CTA covers the whole column chunk)
  const int cols = n * p.g, col = j * p.g + hq % p.g;
  const int cend = min(cols, (col / p.ccols + 1) * p.ccols);
  const int nblk_all = (L - n + (cend - 1) / p.g) / p.BS + 1;
  const int nk = min(p.nkv, (nblk_all + p.kv_chunk - 1) / p.kv_chunk);
  constexpr int V = D / 32;
  float mx = -INFINITY, lsum = 0.f, a[V];
#pragma unroll
  for (int v = 0; v < V; ++v) a[v] = 0.f;
  for (int base = 0; base < nk; base += 32) {
    const int k = base + lane;
    float m = -INFINITY, l = 0.f;
    if (k < nk) {
      m = p.part_ml[(row + k) * 2];
      l = p.part_ml[(row + k) * 2 + 1];
    }
    float cm = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    if (cm == -INFINITY) continue;
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
    const int cnt = min(32, nk - base);
    for (int k0 = 0; k0 < cnt; k0 += 8) {
      float x[8][V], wk[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        wk[u] = __shfl_sync(0xffffffffu, w, (k0 + u) & 31);
        if (k0 + u < cnt && wk[u] != 0.f) {
          const float* o = p.part_o + (row + base + k0 + u) * D;
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
  uint16_t* oh = static_cast<uint16_t*>(p.out) + (q0 + j) * p.o_t + hq * p.o_h + lane * V;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    if constexpr (QBF) oh[v] = __bfloat16_as_ushort(__float2bfloat16_rn(a[v] * inv));
    else oh[v] = __half_as_ushort(__float2half_rn(a[v] * inv));
  }
}

}  // namespace pkv
