// reshape_and_cache (16-bit and fp8-e4m3 pools) and copy_blocks.
//
// reshape_and_cache: each new token's K and V rows go into its slot of the
// sequence's current block ("How Block Paging Operates During Generation",
// "PagedAttention and KV Cache Management"); slot = block * B + offset. One
// thread moves one 16-byte vector of one (token, head) row, so a warp writes
// 512 contiguous bytes of the pool. HBM traffic is 2 * T * Hk * D * e bytes
// read and the same written; at decode sizes the call is launch-latency bound.
//
// copy_blocks: the device half of copy-on-write ("Parallel Sampling & Beam
// Search via Copy-on-Write"): block dst := block src in both pools, bit-exact,
// 16-byte vectors; pairs that would make the result depend on the order of
// the copies are refused (flagged).
//
// swap_blocks_kernel: the device half of preemption by swapping ("Preemption
// and eviction", "Preemption & GPU Swapping"): record i of a page-locked host
// buffer <-> block blocks[i] (its K tile [Hk, B, D] then its V tile), read or
// written by the kernel through the buffer's device mapping, 16-byte vectors:
// a warp moves 512 contiguous bytes of the record.
#pragma once

#include <cuda_fp8.h>

#include "ptx.cuh"

namespace pkv {

struct CacheParams {
  const uint8_t* k;
  const uint8_t* v;
  long long x_s0, x_s1;  // byte strides of k / v rows [T, Hk, D] (same for both)
  long long v_s0, v_s1;
  uint8_t* kc;
  uint8_t* vc;
  long long c_s0, c_s1, c_s2;  // byte strides of the pools [NB, Hk, B, D]
  const long long* slots;
  const float* k_scale;
  const float* v_scale;
  int T, Hk, B, NB;
  int row_vecs;  // 16-byte vectors per (token, head) row of the pools
  int in_bytes;  // bytes of one input row of k / v
};

// The cache writes and block copies are launched as programmatic dependents
// of the kernel before them: they may be resident before it ends, and wait
// for it (griddepcontrol.wait) before touching memory; then they let the
// kernel after them (a decode) start its prologue.

// 16-bit pools: a plain 16-byte copy per thread.
__global__ void reshape_and_cache_kernel(const __grid_constant__ CacheParams p, int* err) {
  pdl_wait();
  pdl_launch_dependents();
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long per_tok = static_cast<long long>(p.Hk) * p.row_vecs;
  if (i >= per_tok * p.T) return;
  const int t = static_cast<int>(i / per_tok);
  const int rem = static_cast<int>(i % per_tok);
  const int h = rem / p.row_vecs, vec = rem % p.row_vecs;
  const long long slot = p.slots[t];
  if (slot < 0) return;
  if (slot >= static_cast<long long>(p.NB) * p.B) {
    if (vec == 0 && h == 0) atomicOr(err, kErrBadSlot);
    return;
  }
  const long long blk = slot / p.B, off = slot % p.B;
  const long long dst = blk * p.c_s0 + h * p.c_s1 + off * p.c_s2 + vec * 16;
  const int4 kv = *reinterpret_cast<const int4*>(p.k + t * p.x_s0 + h * p.x_s1 + vec * 16);
  const int4 vv = *reinterpret_cast<const int4*>(p.v + t * p.v_s0 + h * p.v_s1 + vec * 16);
  *reinterpret_cast<int4*>(p.kc + dst) = kv;
  *reinterpret_cast<int4*>(p.vc + dst) = vv;
}

// fp8 pools: 16 input elements (two 16-byte vectors) -> 16 codes per thread.
template <bool BF16>
__device__ __forceinline__ void widen8(const int4& raw, float (&f)[8]) {
  const uint32_t w[4] = {static_cast<uint32_t>(raw.x), static_cast<uint32_t>(raw.y),
                         static_cast<uint32_t>(raw.z), static_cast<uint32_t>(raw.w)};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if constexpr (BF16) {
      f[2 * j] = __uint_as_float(w[j] << 16);
      f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    } else {
      __half2 hh = *reinterpret_cast<const __half2*>(&w[j]);
      f[2 * j] = __low2float(hh);
      f[2 * j + 1] = __high2float(hh);
    }
  }
}

// 8 widened elements / scale -> 8 e4m3 codes (round to nearest even,
// saturating), the quotient formed with an IEEE fp32 division.
__device__ __forceinline__ uint2 quantise8(const float (&f)[8], float scale) {
  uint32_t w[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 pr = make_float2(__fdiv_rn(f[4 * j + 2 * e], scale),
                                    __fdiv_rn(f[4 * j + 2 * e + 1], scale));
      const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
      word |= static_cast<uint32_t>(q) << (16 * e);
    }
    w[j] = word;
  }
  return make_uint2(w[0], w[1]);
}

template <bool BF16>
__device__ __forceinline__ uint4 quantise16(const int4& a, const int4& b, float scale) {
  float lo[8], hi[8];
  widen8<BF16>(a, lo);
  widen8<BF16>(b, hi);
  const uint2 x = quantise8(lo, scale), y = quantise8(hi, scale);
  return make_uint4(x.x, x.y, y.x, y.y);
}

template <bool BF16>
__global__ void reshape_and_cache_fp8_kernel(const __grid_constant__ CacheParams p, int* err) {
  pdl_wait();
  pdl_launch_dependents();
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long per_tok = static_cast<long long>(p.Hk) * p.row_vecs;
  if (i >= per_tok * p.T) return;
  const int t = static_cast<int>(i / per_tok);
  const int rem = static_cast<int>(i % per_tok);
  const int h = rem / p.row_vecs, vec = rem % p.row_vecs;
  const long long slot = p.slots[t];
  if (slot < 0) return;
  if (slot >= static_cast<long long>(p.NB) * p.B) {
    if (vec == 0 && h == 0) atomicOr(err, kErrBadSlot);
    return;
  }
  const long long blk = slot / p.B, off = slot % p.B;
  const long long dst = blk * p.c_s0 + h * p.c_s1 + off * p.c_s2 + vec * 16;
  const uint8_t* ks = p.k + t * p.x_s0 + h * p.x_s1 + vec * 32;
  const uint8_t* vs = p.v + t * p.v_s0 + h * p.v_s1 + vec * 32;
  const float ksc = p.k_scale[h], vsc = p.v_scale[h];
  *reinterpret_cast<uint4*>(p.kc + dst) =
      quantise16<BF16>(*reinterpret_cast<const int4*>(ks), *reinterpret_cast<const int4*>(ks + 16), ksc);
  *reinterpret_cast<uint4*>(p.vc + dst) =
      quantise16<BF16>(*reinterpret_cast<const int4*>(vs), *reinterpret_cast<const int4*>(vs + 16), vsc);
}

struct CopyParams {
  uint8_t* kc;
  uint8_t* vc;
  long long c_s0, c_s1, c_s2;  // byte strides
  const int* pairs;            // [n][2]
  long long pr_s;              // row stride of pairs (elements)
  int n, Hk, B, NB;
  int row_vecs;                // 16-byte vectors per token row
};

// grid.x = pair, grid.y = chunk of the block's vectors. Every copy of a call
// reads the pool as it was before the call; that holds whatever order the
// CTAs run in as long as no block is written by one pair and read or written
// by another. Each CTA checks its own pair against all the others: a pair
// that shares its destination with another pair's source or destination, or
// whose source is another pair's destination, is not copied and is flagged
// (the other pairs are still copied).
__global__ void copy_blocks_kernel(const __grid_constant__ CopyParams p, int* err) {
  pdl_wait();
  pdl_launch_dependents();
  const int pi = blockIdx.x;
  const int src = p.pairs[pi * p.pr_s], dst = p.pairs[pi * p.pr_s + 1];
  if (src < 0 || src >= p.NB || dst < 0 || dst >= p.NB) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, kErrBadBlock);
    return;
  }
  int clash = 0;
  for (int j = threadIdx.x; j < p.n; j += blockDim.x) {
    if (j == pi) continue;
    const int sj = p.pairs[j * p.pr_s], dj = p.pairs[j * p.pr_s + 1];
    clash |= (sj == dst) | (dj == dst) | (dj == src);
  }
  if (__syncthreads_or(clash)) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, kErrBadCopy);
    return;
  }
  const int per_head = p.B * p.row_vecs;
  const int total = p.Hk * per_head;
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < total; v += gridDim.y * blockDim.x) {
    const int h = v / per_head, rem = v % per_head;
    const int row = rem / p.row_vecs, vec = rem % p.row_vecs;
    const long long o = h * p.c_s1 + row * p.c_s2 + vec * 16;
    const long long so = src * p.c_s0 + o, d = dst * p.c_s0 + o;
    *reinterpret_cast<int4*>(p.kc + d) = *reinterpret_cast<const int4*>(p.kc + so);
    *reinterpret_cast<int4*>(p.vc + d) = *reinterpret_cast<const int4*>(p.vc + so);
  }
}

struct SwapParams {
  uint8_t* kc;
  uint8_t* vc;
  long long c_s0, c_s1, c_s2;  // byte strides of the pools [NB, Hk, B, D]
  uint8_t* host;               // device address of the host records
  const int* blocks;
  long long bl_s;
  int n, Hk, B, NB;
  int row_vecs;         // 16-byte vectors per (head, token) row
  long long rec_bytes;  // bytes of one record: K tile then V tile
};

template <bool kOut>
__global__ void swap_blocks_kernel(const __grid_constant__ SwapParams p, int* err) {
  const int i = blockIdx.x;
  const int blk = p.blocks[i * p.bl_s];
  if (blk < 0 || blk >= p.NB) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, kErrBadBlock);
    return;
  }
  const int per_head = p.B * p.row_vecs;
  const int total = p.Hk * per_head;  // vectors per tile
  uint8_t* rec = p.host + static_cast<long long>(i) * p.rec_bytes;
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < total; v += gridDim.y * blockDim.x) {
    const int h = v / per_head, rem = v % per_head;
    const int row = rem / p.row_vecs, vec = rem % p.row_vecs;
    const long long o = blk * p.c_s0 + h * p.c_s1 + row * p.c_s2 + vec * 16;
    int4* rk = reinterpret_cast<int4*>(rec + static_cast<long long>(v) * 16);
    int4* rv = reinterpret_cast<int4*>(rec + (static_cast<long long>(total) + v) * 16);
    if constexpr (kOut) {
      *rk = *reinterpret_cast<const int4*>(p.kc + o);
      *rv = *reinterpret_cast<const int4*>(p.vc + o);
    } else {
      *reinterpret_cast<int4*>(p.kc + o) = *rk;
      *reinterpret_cast<int4*>(p.vc + o) = *rv;
    }
  }
}

}  // namespace pkv
