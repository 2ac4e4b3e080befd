// C ABI of libpagedkv.so (declared in include/pagedkv.h): argument checks,
// TMA tensor-map encoding, workspace management and kernel dispatch for the
// decode, cache-write and block-copy kernels. The host allocator lives in
// allocator.cpp.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/pagedkv.h"
#include "cache_ops.cuh"
#include "cascade.cuh"
#include "prefill.cuh"
#include "prefill_tc.cuh"
#include "prefill_tc2.cuh"
#include "decode.cuh"

namespace pkv {

// Per-device error word the kernels OR their device-check bits into.
__device__ int g_pkv_err;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool init = false;
  int sms = 0;
  int* err = nullptr;  // device address of g_pkv_err
  void* ws = nullptr;  // library-owned decode workspace
  size_t ws_bytes = 0;
  void* cas = nullptr;  // library-owned prefix-aware decode partials
  size_t cas_bytes = 0;
  void* pre = nullptr;  // library-owned multi-token partials
  size_t pre_bytes = 0;
  int* ord = nullptr;   // library-owned sequence order for the tensor-core multi-token kernels
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return PKV_ERR_UNSUPPORTED;
  return PKV_OK;
}

// Device properties and the error word's address, once per device (with
// that device current).
int device_state(int dev, DeviceState** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return PKV_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pkv_err) != cudaSuccess) return PKV_ERR_CUDA;
    d.err = static_cast<int*>(p);
    d.init = true;
  }
  *out = &d;
  return PKV_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int elem_bytes(int dt) {
  switch (dt) {
    case PKV_F16:
    case PKV_BF16: return 2;
    case PKV_FP8_E4M3: return 1;
    case PKV_I32:
    case PKV_F32: return 4;
    case PKV_I64: return 8;
    default: return 0;
  }
}

bool well_formed(const pkv_tensor* t, int ndim, int dtype) {
  if (!t || t->ndim != ndim || t->dtype != dtype) return false;
  for (int i = 0; i < ndim; ++i)
    if (t->shape[i] < 0) return false;
  if (ndim > 0 && t->shape[ndim - 1] > 1 && t->stride[ndim - 1] != 1) return false;
  for (int i = 0; i < ndim; ++i)
    if (t->stride[i] < 0) return false;
  bool empty = false;
  for (int i = 0; i < ndim; ++i) empty |= t->shape[i] == 0;
  return empty || t->data != nullptr;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Pool [NB, Hk, B, D]: innermost contiguous, strides non-decreasing outward,
// byte strides multiples of 16, base 16-byte aligned.
bool pool_ok(const pkv_tensor* t, int dtype) {
  if (!well_formed(t, 4, dtype)) return false;
  const int64_t eb = elem_bytes(dtype);
  const int64_t* sh = t->shape;
  const int64_t* st = t->stride;
  if (st[3] != 1) return false;
  if (st[2] < sh[3] || st[1] < sh[2] * st[2] || st[0] < sh[1] * st[1]) return false;
  for (int i = 0; i < 3; ++i)
    if ((st[i] * eb) % 16 != 0) return false;
  return aligned(t->data, 16);
}

bool same_shape(const pkv_tensor* a, const pkv_tensor* b) {
  if (a->ndim != b->ndim) return false;
  for (int i = 0; i < a->ndim; ++i)
    if (a->shape[i] != b->shape[i]) return false;
  return true;
}

int encode_pool_map(CUtensorMap* map, const pkv_tensor* pool, int dtype) {
  auto fn = encode_fn();
  if (!fn) return PKV_ERR_CUDA;
  const int eb = elem_bytes(dtype);
  const int D = static_cast<int>(pool->shape[3]);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(pool->shape[2]),
                        static_cast<cuuint64_t>(pool->shape[1]),
                        static_cast<cuuint64_t>(pool->shape[0])};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(pool->stride[2] * eb),
                           static_cast<cuuint64_t>(pool->stride[1] * eb),
                           static_cast<cuuint64_t>(pool->stride[0] * eb)};
  const int epr = 128 / eb;
  cuuint32_t box[4] = {static_cast<cuuint32_t>(D < epr ? D : epr),
                       static_cast<cuuint32_t>(pool->shape[2]), 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUtensorMapDataType ty = dtype == PKV_F16    ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                           : dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                               : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(map, ty, 4, pool->data, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PKV_OK : PKV_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Decode kernel registry
// ---------------------------------------------------------------------------

struct DecodeLaunch {
  void (*kernel)(DecodeParams);
  void (*merge)(DecodeParams);
  int threads;
  int smem;
  int nc;
  int occ[kMaxDevices];  // resident CTAs per SM, 0 = not queried yet
};

template <int CK, bool QBF, int D, int BS, int NC, int NS, int IB = 1>
DecodeLaunch* decode_entry() {
  static DecodeLaunch e = {&decode_kernel<CK, QBF, D, BS, NC, NS, IB>,
                           &decode_merge_kernel<QBF, D>,
                           NC * 32,
                           DecodeCfg<CK, QBF, D, BS, NC, NS, IB>::SMEM,
                           NC,
                           {0}};
  return &e;
}

// Warps per CTA (NC), ring stages per warp (NS) and blocks per work item
// (IB), measured on B200. Two CTAs of ~96 KB share an SM where a stage is
// 8 KB or less: 16-bit, D = 128, 16-token blocks run 4 warps x 3 stages (the
// same 24 stages in flight per SM as 3 warps x 4, but a third more, shorter
// warp ranges: long_skewed 537 -> 492 us, llama3_8b 112.5 -> 110.7 us);
// D = 64 with 4 warps x 6 stages of 4 KB; 32-token 16-bit blocks use 3 warps
// x 2 stages of 16 KB (two CTAs per SM: 475 -> 457 us on long_skewed with
// 32-token blocks against 4 x 3, one CTA per SM). fp8 items take two 16-token blocks
// (32 tokens, 8 KB stages): the widening makes fp8 issue-bound, and larger
// items halve the per-item overhead.
DecodeLaunch* pick_decode(int ck, bool qbf, int D, int BS) {
  constexpr int NC = 4;
  if (ck == kCacheBF16) {
    if (D == 128 && BS == 16) return decode_entry<kCacheBF16, true, 128, 16, NC, 3>();
    if (D == 128 && BS == 32) return decode_entry<kCacheBF16, true, 128, 32, 3, 2>();
    if (D == 64 && BS == 16) return decode_entry<kCacheBF16, true, 64, 16, NC, 6>();
    if (D == 64 && BS == 32) return decode_entry<kCacheBF16, true, 64, 32, NC, 3>();
  } else if (ck == kCacheF16) {
    if (D == 128 && BS == 16) return decode_entry<kCacheF16, false, 128, 16, NC, 3>();
    if (D == 128 && BS == 32) return decode_entry<kCacheF16, false, 128, 32, 3, 2>();
    if (D == 64 && BS == 16) return decode_entry<kCacheF16, false, 64, 16, NC, 6>();
    if (D == 64 && BS == 32) return decode_entry<kCacheF16, false, 64, 32, NC, 3>();
  } else if (ck == kCacheE4M3 && D == 128) {
    if (qbf) {
      if (BS == 16) return decode_entry<kCacheE4M3, true, 128, 16, NC, 3, 2>();
      if (BS == 32) return decode_entry<kCacheE4M3, true, 128, 32, NC, 3>();
    } else {
      if (BS == 16) return decode_entry<kCacheE4M3, false, 128, 16, NC, 3, 2>();
      if (BS == 32) return decode_entry<kCacheE4M3, false, 128, 32, NC, 3>();
    }
  }
  return nullptr;
}

int decode_grid(DecodeLaunch* e, int dev, int sms, int* grid) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (e->occ[dev] == 0) {
    if (cudaFuncSetAttribute(e->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, e->smem) !=
        cudaSuccess)
      return PKV_ERR_CUDA;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, e->kernel, e->threads, e->smem) !=
            cudaSuccess ||
        occ < 1)
      return PKV_ERR_CUDA;
    e->occ[dev] = occ;
  }
  *grid = e->occ[dev] * sms;
  return PKV_OK;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch as a programmatic dependent of the kernel before it in the stream
// (the kernel waits for it with griddepcontrol.wait before touching memory).
template <typename P>
int launch_dependent(void (*kern)(P, int*), dim3 grid, dim3 block, cudaStream_t stream, const P& p,
                     int* err) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, err) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Decode workspace: header (total items, steal-slot pool counter), range
// words, steal records, last-piece descriptors, and fp32 partial slots (two
// per warp for its own range, `pool` more for steals). The range words and
// the pool counter must be zero before a call (every call leaves them zero
// again) and steal records are recognised by the call's tag, so these
// regions sit at the same offsets, with the same sizes, for every kernel
// configuration (sized for kWordsPerSM warps per SM, more than any
// configuration has): no configuration's scratch ever lands in another's
// claim state or steal records.
constexpr int kWordsPerSM = 16;

struct WsLayout {
  size_t hdr, pool, words, steal, desc, rlo, adapt, part_o, part_ml, total;
  size_t cap;  // warps the fixed regions are sized for
  int pool_slots;
};

size_t slot_bytes(int g, int D) { return static_cast<size_t>(g) * (D + 2) * 4; }

WsLayout ws_layout(int sms, int nwt, int g, int D, int pool_slots) {
  WsLayout l;
  l.hdr = 0;
  l.pool = 64;
  l.words = 256;
  size_t cap = static_cast<size_t>(kWordsPerSM) * sms;
  if (cap < static_cast<size_t>(nwt)) cap = nwt;
  l.steal = round_up(l.words + cap * 8, 256);
  l.desc = round_up(l.steal + cap * kMaxSteals * 16, 256);
  l.rlo = round_up(l.desc + cap * (1 + kMaxSteals) * 16, 256);
  // adaptive partition: its nwt word, then part, rtime and wgt [cap] each
  l.adapt = round_up(l.rlo + (cap + 1) * 8, 256);
  l.cap = cap;
  l.part_o = round_up(l.adapt + 16 + cap * 12, 256);
  const size_t slots = 2 * static_cast<size_t>(nwt) + pool_slots;
  l.part_ml = round_up(l.part_o + slots * g * D * 4, 256);
  l.total = round_up(l.part_ml + slots * g * 2 * 4, 256);
  l.pool_slots = pool_slots;
  return l;
}

// Default: room for two steals per warp on average.
WsLayout ws_default(int sms, int nwt, int g, int D) {
  return ws_layout(sms, nwt, g, D, 4 * nwt);
}

// The largest layout that fits in `bytes` (fewer steal slots), or one whose
// total exceeds `bytes` when even no steal slots fit.
WsLayout ws_fit(int sms, int nwt, int g, int D, size_t bytes) {
  const WsLayout full = ws_default(sms, nwt, g, D);
  if (full.total <= bytes) return full;
  const WsLayout base = ws_layout(sms, nwt, g, D, 0);
  if (base.total > bytes) return base;
  int pool = static_cast<int>((bytes - base.total) / slot_bytes(g, D)) & ~1;
  while (pool > 0 && ws_layout(sms, nwt, g, D, pool).total > bytes) pool -= 2;
  return ws_layout(sms, nwt, g, D, pool);
}

std::atomic<unsigned> g_call_tag{1};

int next_tag() {
  for (;;) {
    const unsigned t = g_call_tag.fetch_add(1);
    if (static_cast<int>(t) != 0) return static_cast<int>(t);
  }
}

struct DecodeArgs {
  const pkv_tensor *q, *kc, *vc, *ks, *vs, *bt, *cl;
  int Hk;
  float scale;
  int BS;
  pkv_tensor* out;
};

// Checks shapes/types and resolves the kernel. On PKV_OK, *entry is set, or
// left NULL when there is nothing to compute (S == 0).
int check_decode(const DecodeArgs& a, bool fp8, int* ck_out, DecodeLaunch** entry) {
  *entry = nullptr;
  if (!a.q || !a.kc || !a.vc || !a.bt || !a.cl || !a.out) return PKV_ERR_INVALID_ARG;
  const int qdt = a.q->dtype;
  if (qdt != PKV_F16 && qdt != PKV_BF16) return PKV_ERR_INVALID_ARG;
  if (!well_formed(a.q, 3, qdt) || !well_formed(a.out, 3, qdt) || !same_shape(a.q, a.out))
    return PKV_ERR_INVALID_ARG;
  const int cdt = fp8 ? PKV_FP8_E4M3 : qdt;
  if (!pool_ok(a.kc, cdt) || !pool_ok(a.vc, cdt) || !same_shape(a.kc, a.vc))
    return PKV_ERR_INVALID_ARG;
  const int64_t S = a.q->shape[0], Hq = a.q->shape[1], D = a.q->shape[2];
  const int64_t NB = a.kc->shape[0], Hk = a.kc->shape[1], BS = a.kc->shape[2];
  if (a.kc->shape[3] != D || Hk != a.Hk || BS != a.BS || Hk <= 0 || Hq % Hk != 0)
    return PKV_ERR_INVALID_ARG;
  if (!well_formed(a.bt, 2, PKV_I32) || a.bt->shape[0] != S) return PKV_ERR_INVALID_ARG;
  if (!well_formed(a.cl, 1, PKV_I32) || a.cl->shape[0] != S) return PKV_ERR_INVALID_ARG;
  if (S > 0 && a.cl->stride[0] != 1) return PKV_ERR_INVALID_ARG;
  if (!std::isfinite(a.scale)) return PKV_ERR_INVALID_ARG;
  if (fp8) {
    if (!a.ks || !a.vs || !well_formed(a.ks, 1, PKV_F32) || !well_formed(a.vs, 1, PKV_F32) ||
        a.ks->shape[0] != Hk || a.vs->shape[0] != Hk || a.ks->stride[0] != 1 ||
        a.vs->stride[0] != 1)
      return PKV_ERR_INVALID_ARG;
  }
  // q rows are read as 4- (16-bit cache) or 8-byte (fp8 cache) words
  const int qa = fp8 ? 4 : 2;
  if (S > 0 && (a.q->stride[0] % qa || a.q->stride[1] % qa || !aligned(a.q->data, 2 * qa)))
    return PKV_ERR_INVALID_ARG;
  const int64_t g = Hq / Hk;
  if (g > 8 || (D != 64 && D != 128) || (BS != 16 && BS != 32) || (fp8 && D != 128))
    return PKV_ERR_UNSUPPORTED;
  if (NB > INT32_MAX || S > INT32_MAX || a.bt->shape[1] > INT32_MAX / 32)
    return PKV_ERR_UNSUPPORTED;
  if (S == 0) return PKV_OK;
  if (a.bt->shape[1] < 1 || NB < 1) return PKV_ERR_INVALID_ARG;
  const int ck = fp8 ? kCacheE4M3 : (qdt == PKV_BF16 ? kCacheBF16 : kCacheF16);
  *ck_out = ck;
  *entry = pick_decode(ck, qdt == PKV_BF16, static_cast<int>(D), static_cast<int>(BS));
  return *entry ? PKV_OK : PKV_ERR_UNSUPPORTED;
}

// Prefix-aware decode: table entries each sequence skips, and where the
// sequences with a prefix leave their partials.
struct CascadeTail {
  const int* skip;
  float* o;
  float* ml;
};

// Launch decode + merge. lib_ws: use (and grow) the library's workspace for
// this device; otherwise `ws` is the caller's. fit: shrink the steal-slot pool
// to fit ws_bytes; clear: zero the claim state first (callers that cannot
// vouch for it); fixed_split: no work stealing (identical calls give
// identical bits).
int launch_decode(const DecodeArgs& a, bool fp8, void* ws, size_t ws_bytes, bool lib_ws,
                  cudaStream_t stream, bool fit = false, bool clear = false,
                  const CascadeTail* tail = nullptr, bool fixed_split = false) {
  int ck = 0;
  DecodeLaunch* e = nullptr;
  int st = check_decode(a, fp8, &ck, &e);
  if (st != PKV_OK || !e) return st;
  int dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  DeviceState* ds;
  if ((st = device_state(dev, &ds)) != PKV_OK) return st;
  int grid;
  if ((st = decode_grid(e, dev, ds->sms, &grid)) != PKV_OK) return st;
  const int nwt = grid * e->nc;
  const int g = static_cast<int>(a.q->shape[1] / a.Hk);
  const int D = static_cast<int>(a.q->shape[2]);
  if (nwt > kWordsPerSM * ds->sms) return PKV_ERR_UNSUPPORTED;
  const WsLayout L = fit ? ws_fit(ds->sms, nwt, g, D, ws_bytes) : ws_default(ds->sms, nwt, g, D);
  if (lib_ws) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (ds->ws_bytes < L.total) {
      if (ds->ws) cudaFree(ds->ws);
      ds->ws = nullptr;
      ds->ws_bytes = 0;
      if (cudaMalloc(&ds->ws, L.total) != cudaSuccess) return PKV_ERR_CUDA;
      // zeroed on the call's stream, so this launch sees it zeroed
      if (cudaMemsetAsync(ds->ws, 0, L.total, stream) != cudaSuccess) return PKV_ERR_CUDA;
      ds->ws_bytes = L.total;
    }
    ws = ds->ws;
    ws_bytes = ds->ws_bytes;
  }
  if (fit && L.total > ws_bytes) return PKV_ERR_SCRATCH_LIMIT;  // even with no steal slots
  if (!ws || ws_bytes < L.total || !aligned(ws, 16)) return PKV_ERR_WORKSPACE;
  if (clear && cudaMemsetAsync(ws, 0, L.steal, stream) != cudaSuccess) return PKV_ERR_CUDA;

  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  const int cdt = fp8 ? PKV_FP8_E4M3 : a.q->dtype;
  if ((st = encode_pool_map(&p.tmk, a.kc, cdt)) != PKV_OK) return st;
  if ((st = encode_pool_map(&p.tmv, a.vc, cdt)) != PKV_OK) return st;
  p.q = a.q->data;
  p.q_s = a.q->stride[0];
  p.q_h = a.q->stride[1];
  p.out = a.out->data;
  p.o_s = a.out->stride[0];
  p.o_h = a.out->stride[1];
  p.tables = static_cast<const int*>(a.bt->data);
  p.t_s = a.bt->stride[0];
  p.lens = static_cast<const int*>(a.cl->data);
  p.k_scale = fp8 ? static_cast<const float*>(a.ks->data) : nullptr;
  p.v_scale = fp8 ? static_cast<const float*>(a.vs->data) : nullptr;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.S = static_cast<int>(a.q->shape[0]);
  p.Hk = a.Hk;
  p.g = g;
  p.MB = static_cast<int>(a.bt->shape[1]);
  p.NB = static_cast<int>(a.kc->shape[0]);
  p.nwt = nwt;
  p.tag = next_tag();
  p.steal = fixed_split ? 0 : 1;
  // The adaptive partition pays off where the per-warp speed differences
  // repeat from call to call: the fp8 kernel is issue-bound and a range of
  // many short sequences is slower than one of few long ones. With fewer
  // (sequence, kv head) units than warp ranges every range lies inside one
  // or two long units, and the speed differences follow the SMs the CTAs
  // land on, which change between calls; so do those of the HBM-bound
  // 16-bit kernels. Equal ranges plus stealing do better there (fp8
  // llama3_8b shape, 512 units for 1184 ranges: 65.7 against 68.8 us).
  const long long units = static_cast<long long>(p.S) * a.Hk;
  p.adapt = fp8 && !fixed_split && nwt <= 128 * kAdaptPer && units >= nwt ? 1 : 0;
  p.pool_slots = L.pool_slots;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.hdr = reinterpret_cast<long long*>(w + L.hdr);
  p.err = ds->err;
  p.words = reinterpret_cast<unsigned long long*>(w + L.words);
  p.pool = reinterpret_cast<unsigned*>(w + L.pool);
  p.steal_info = reinterpret_cast<int4*>(w + L.steal);
  p.desc = reinterpret_cast<int4*>(w + L.desc);
  p.rlo = reinterpret_cast<long long*>(w + L.rlo);
  {
    int* an = reinterpret_cast<int*>(w + L.adapt);
    const size_t cap = L.cap;
    unsigned* part = reinterpret_cast<unsigned*>(w + L.adapt + 16);
    p.part_nwt = an;
    p.part_nwt_w = an;
    p.part = part;
    p.part_w = part;
    p.rtime = reinterpret_cast<float*>(part + cap);
    p.wgt = p.rtime + cap;
  }
  p.part_o = reinterpret_cast<float*>(w + L.part_o);
  p.part_ml = reinterpret_cast<float*>(w + L.part_ml);
  if (tail) {
    p.skip = tail->skip;
    p.cas_o = tail->o;
    p.cas_ml = tail->ml;
  }

  // Both kernels are launched as programmatic dependents of the kernel
  // before them in the stream: their CTAs can be resident before it ends and
  // start work the moment it has (griddepcontrol.wait), hiding launch gaps.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(e->threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(e->smem);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, e->kernel, p) != cudaSuccess) return PKV_ERR_CUDA;
  cfg.gridDim = dim3(static_cast<unsigned>(nwt));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, e->merge, p) != cudaSuccess) return PKV_ERR_CUDA;
  return PKV_OK;
}

// ---------------------------------------------------------------------------
// Prefix-aware decode
// ---------------------------------------------------------------------------

struct CascadeLaunch {
  void (*prefix)(CascadeParams);
  void (*merge)(CascadeParams);
  int smem;
  bool attr_set[kMaxDevices];
};

template <bool QBF, int D, int BS, bool FP8 = false>
CascadeLaunch* cascade_entry() {
  constexpr int NS = 4;
  static CascadeLaunch e = {&cascade_prefix_kernel<QBF, D, BS, NS, FP8>, &cascade_merge_kernel<QBF, D>,
                            PrefixCfg<QBF, D, BS, NS, FP8>::SMEM, {false}};
  return &e;
}

CascadeLaunch* pick_cascade(bool qbf, int D, int BS, bool fp8) {
  if (fp8) {  // e4m3 pools, D = 128
    if (D != 128) return nullptr;
    if (qbf) return BS == 16 ? cascade_entry<true, 128, 16, true>() : cascade_entry<true, 128, 32, true>();
    return BS == 16 ? cascade_entry<false, 128, 16, true>() : cascade_entry<false, 128, 32, true>();
  }
  if (qbf) {
    if (D == 128 && BS == 16) return cascade_entry<true, 128, 16>();
    if (D == 128 && BS == 32) return cascade_entry<true, 128, 32>();
    if (D == 64 && BS == 16) return cascade_entry<true, 64, 16>();
    if (D == 64 && BS == 32) return cascade_entry<true, 64, 32>();
  } else {
    if (D == 128 && BS == 16) return cascade_entry<false, 128, 16>();
    if (D == 128 && BS == 32) return cascade_entry<false, 128, 32>();
    if (D == 64 && BS == 16) return cascade_entry<false, 64, 16>();
    if (D == 64 && BS == 32) return cascade_entry<false, 64, 32>();
  }
  return nullptr;
}

int launch_cascade(const DecodeArgs& a, bool fp8, const pkv_tensor* pblk, const pkv_tensor* gstart,
                   const pkv_tensor* gmem, int G, int max_members, int max_prefix,
                   cudaStream_t stream) {
  int ck = 0;
  DecodeLaunch* e = nullptr;
  int st = check_decode(a, fp8, &ck, &e);
  if (st != PKV_OK) return st;
  if (!pblk || !gstart || !gmem || G < 0 || max_members < 0 || max_prefix < 0)
    return PKV_ERR_INVALID_ARG;
  const int64_t S = a.q->shape[0];
  if (!well_formed(pblk, 1, PKV_I32) || pblk->shape[0] != S || (S > 0 && pblk->stride[0] != 1))
    return PKV_ERR_INVALID_ARG;
  if (!well_formed(gstart, 1, PKV_I32) || gstart->shape[0] != G + 1 || gstart->stride[0] != 1)
    return PKV_ERR_INVALID_ARG;
  if (!well_formed(gmem, 1, PKV_I32) || (gmem->shape[0] > 0 && gmem->stride[0] != 1) ||
      gmem->shape[0] > S || gmem->shape[0] > INT32_MAX)
    return PKV_ERR_INVALID_ARG;
  const int M = static_cast<int>(gmem->shape[0]);
  if (!e) return PKV_OK;  // S == 0
  if (max_prefix > a.bt->shape[1] || max_members > S || (G > 0 && (max_members < 1 || M < 1)))
    return PKV_ERR_INVALID_ARG;
  const int D = static_cast<int>(a.q->shape[2]);
  const int g = static_cast<int>(a.q->shape[1] / a.Hk);
  CascadeLaunch* ce = pick_cascade(a.q->dtype == PKV_BF16, D, a.BS, fp8);
  if (!ce) return PKV_ERR_UNSUPPORTED;
  int dev;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  DeviceState* ds;
  if ((st = device_state(dev, &ds)) != PKV_OK) return st;

  // prefix chunks: about two CTAs per SM over all (group, head, column chunk)
  const int ncc = std::max(1, (max_members * g + kCasCols - 1) / kCasCols);
  const long long pairs = static_cast<long long>(G) * a.Hk * ncc * std::max(max_prefix, 1);
  int cb = static_cast<int>((pairs + 2LL * ds->sms - 1) / (2LL * ds->sms));
  cb = std::min(std::max(cb, std::min(4, std::max(max_prefix, 1))), kCasMaxChunk);
  const int nkc = std::max(1, (max_prefix + cb - 1) / cb);
  const long long items = static_cast<long long>(G) * a.Hk * ncc * nkc;
  const int Hq = a.Hk * g;
  const size_t suf_o = 0;
  const size_t suf_ml = round_up(suf_o + static_cast<size_t>(S) * Hq * D * 4, 256);
  const size_t pre_o = round_up(suf_ml + static_cast<size_t>(S) * Hq * 2 * 4, 256);
  const size_t pre_ml = round_up(pre_o + static_cast<size_t>(items) * kCasCols * D * 4, 256);
  const size_t total = round_up(pre_ml + static_cast<size_t>(items) * kCasCols * 2 * 4, 256);
  if (nkc > 65535 || ncc > 65535 || static_cast<long long>(G) * a.Hk > 65535)
    return PKV_ERR_UNSUPPORTED;
  uint8_t* cw;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (ds->cas_bytes < total) {
      if (ds->cas) cudaFree(ds->cas);
      ds->cas = nullptr;
      ds->cas_bytes = 0;
      if (cudaMalloc(&ds->cas, total) != cudaSuccess) return PKV_ERR_CUDA;
      ds->cas_bytes = total;
    }
    cw = static_cast<uint8_t*>(ds->cas);
    if (!ce->attr_set[dev]) {
      if (cudaFuncSetAttribute(ce->prefix, cudaFuncAttributeMaxDynamicSharedMemorySize, ce->smem) !=
          cudaSuccess)
        return PKV_ERR_CUDA;
      ce->attr_set[dev] = true;
    }
  }
  CascadeTail tail{static_cast<const int*>(pblk->data), reinterpret_cast<float*>(cw + suf_o),
                   reinterpret_cast<float*>(cw + suf_ml)};
  if ((st = launch_decode(a, fp8, nullptr, 0, true, stream, false, false, &tail)) != PKV_OK)
    return st;
  if (G == 0 || M == 0) return PKV_OK;

  CascadeParams p;
  std::memset(&p, 0, sizeof(p));
  const int cdt = fp8 ? PKV_FP8_E4M3 : a.q->dtype;
  if ((st = encode_pool_map(&p.tmk, a.kc, cdt)) != PKV_OK) return st;
  if ((st = encode_pool_map(&p.tmv, a.vc, cdt)) != PKV_OK) return st;
  p.q = a.q->data;
  p.q_s = a.q->stride[0];
  p.q_h = a.q->stride[1];
  p.out = a.out->data;
  p.o_s = a.out->stride[0];
  p.o_h = a.out->stride[1];
  p.tables = static_cast<const int*>(a.bt->data);
  p.t_s = a.bt->stride[0];
  p.k_scale = fp8 ? static_cast<const float*>(a.ks->data) : nullptr;
  p.v_scale = fp8 ? static_cast<const float*>(a.vs->data) : nullptr;
  p.prefix_blocks = static_cast<const int*>(pblk->data);
  p.group_start = static_cast<const int*>(gstart->data);
  p.members = static_cast<const int*>(gmem->data);
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.S = static_cast<int>(S);
  p.Hk = a.Hk;
  p.g = g;
  p.NB = static_cast<int>(a.kc->shape[0]);
  p.MB = static_cast<int>(a.bt->shape[1]);
  p.G = G;
  p.M = M;
  p.ncc = ncc;
  p.nkc = nkc;
  p.cb = cb;
  p.err = ds->err;
  p.pre_o = reinterpret_cast<float*>(cw + pre_o);
  p.pre_ml = reinterpret_cast<float*>(cw + pre_ml);
  p.suf_o = reinterpret_cast<const float*>(cw + suf_o);
  p.suf_ml = reinterpret_cast<const float*>(cw + suf_ml);

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nkc), static_cast<unsigned>(ncc),
                     static_cast<unsigned>(G * a.Hk));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = static_cast<size_t>(ce->smem);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, ce->prefix, p) != cudaSuccess) return PKV_ERR_CUDA;
  const long long warps = static_cast<long long>(max_members) * Hq;
  if ((warps + 3) / 4 > INT32_MAX || G > 65535) return PKV_ERR_UNSUPPORTED;
  cfg.gridDim = dim3(static_cast<unsigned>((warps + 3) / 4), static_cast<unsigned>(G));
  cfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&cfg, ce->merge, p) != cudaSuccess) return PKV_ERR_CUDA;
  return PKV_OK;
}

// ---------------------------------------------------------------------------
// Multi-token (causal) paged attention
// ---------------------------------------------------------------------------

struct PrefillLaunch {
  void (*kernel)(PrefillParams);
  void (*merge)(PrefillParams);
  int threads, smem, cols;
  bool attr_set[kMaxDevices];
};

template <bool QBF, int D, int BS, int NW, bool FP8 = false>
PrefillLaunch* prefill_entry() {
  constexpr int NS = 4;
  static PrefillLaunch e = {&prefill_kernel<QBF, D, BS, NS, NW, FP8>, &prefill_merge_kernel<QBF, D>, NW * 32,
                            PrefillCfg<QBF, D, BS, NS, NW, FP8>::SMEM, NW * 16, {false}};
  return &e;
}

template <bool QBF, int D, int BS, bool FP8 = false>
PrefillLaunch* prefill_by_cols(int cols) {
  if (cols <= 16) return prefill_entry<QBF, D, BS, 1, FP8>();
  if (cols <= 32) return prefill_entry<QBF, D, BS, 2, FP8>();
  return prefill_entry<QBF, D, BS, 4, FP8>();
}

PrefillLaunch* pick_prefill(bool qbf, int D, int BS, int cols, bool fp8) {
  if (fp8) {  // e4m3 pools, D = 128
    if (D != 128) return nullptr;
    if (qbf) return BS == 16 ? prefill_by_cols<true, 128, 16, true>(cols) : prefill_by_cols<true, 128, 32, true>(cols);
    return BS == 16 ? prefill_by_cols<false, 128, 16, true>(cols) : prefill_by_cols<false, 128, 32, true>(cols);
  }
  if (qbf) {
    if (D == 128 && BS == 16) return prefill_by_cols<true, 128, 16>(cols);
    if (D == 128 && BS == 32) return prefill_by_cols<true, 128, 32>(cols);
    if (D == 64 && BS == 16) return prefill_by_cols<true, 64, 16>(cols);
    if (D == 64 && BS == 32) return prefill_by_cols<true, 64, 32>(cols);
  } else {
    if (D == 128 && BS == 16) return prefill_by_cols<false, 128, 16>(cols);
    if (D == 128 && BS == 32) return prefill_by_cols<false, 128, 32>(cols);
    if (D == 64 && BS == 16) return prefill_by_cols<false, 64, 16>(cols);
    if (D == 64 && BS == 32) return prefill_by_cols<false, 64, 32>(cols);
  }
  return nullptr;
}

// Tensor-core (tcgen05) variants, D = 128: prefill_tc2_kernel (two 128-row
// tiles per CTA) where a (sequence, head) may have more than 128 rows,
// prefill_tc_kernel (one tile) otherwise.
struct PrefillTcLaunch {
  void (*kernel)(PrefillParams);
  int smem;
  int rows;     // query rows per CTA
  int threads;
  bool attr_set[kMaxDevices];
};

template <bool QBF, int BS>
PrefillTcLaunch* prefill_tc_entry() {
  static PrefillTcLaunch e = {&prefill_tc_kernel<QBF, BS>, PrefillTcCfg<BS>::SMEM, PrefillTcCfg<BS>::ROWS,
                              PrefillTcCfg<BS>::THREADS, {false}};
  return &e;
}
template <bool QBF, int BS>
PrefillTcLaunch* prefill_tc2_entry() {
  static PrefillTcLaunch e = {&prefill_tc2_kernel<QBF, BS>, PrefillTc2Cfg<BS>::SMEM, PrefillTc2Cfg<BS>::ROWS,
                              PrefillTc2Cfg<BS>::THREADS, {false}};
  return &e;
}

PrefillTcLaunch* pick_prefill_tc(bool qbf, int BS, int cols) {
  if (cols > 128) {
    if (qbf) return BS == 16 ? prefill_tc2_entry<true, 16>() : prefill_tc2_entry<true, 32>();
    return BS == 16 ? prefill_tc2_entry<false, 16>() : prefill_tc2_entry<false, 32>();
  }
  if (qbf) return BS == 16 ? prefill_tc_entry<true, 16>() : prefill_tc_entry<true, 32>();
  return BS == 16 ? prefill_tc_entry<false, 16>() : prefill_tc_entry<false, 32>();
}

int launch_prefill(const pkv_tensor* q, const pkv_tensor* kc, const pkv_tensor* vc,
                   const pkv_tensor* ks, const pkv_tensor* vs, bool fp8,
                   const pkv_tensor* bt, const pkv_tensor* cl, const pkv_tensor* qs, int max_q,
                   int Hk, float scale, int BS, pkv_tensor* out, cudaStream_t stream) {
  if (!q || !kc || !vc || !bt || !cl || !qs || !out) return PKV_ERR_INVALID_ARG;
  const int qdt = q->dtype;
  if (qdt != PKV_F16 && qdt != PKV_BF16) return PKV_ERR_INVALID_ARG;
  if (!well_formed(q, 3, qdt) || !well_formed(out, 3, qdt) || !same_shape(q, out))
    return PKV_ERR_INVALID_ARG;
  const int cdt = fp8 ? PKV_FP8_E4M3 : qdt;
  if (!pool_ok(kc, cdt) || !pool_ok(vc, cdt) || !same_shape(kc, vc)) return PKV_ERR_INVALID_ARG;
  if (fp8 && (!ks || !vs || !well_formed(ks, 1, PKV_F32) || !well_formed(vs, 1, PKV_F32) ||
              ks->shape[0] != Hk || vs->shape[0] != Hk || ks->stride[0] != 1 || vs->stride[0] != 1))
    return PKV_ERR_INVALID_ARG;
  const int64_t T = q->shape[0], Hq = q->shape[1], D = q->shape[2];
  const int64_t NB = kc->shape[0];
  if (kc->shape[1] != Hk || kc->shape[2] != BS || kc->shape[3] != D || Hk <= 0 || Hq % Hk != 0)
    return PKV_ERR_INVALID_ARG;
  if (!well_formed(bt, 2, PKV_I32) || !well_formed(cl, 1, PKV_I32)) return PKV_ERR_INVALID_ARG;
  const int64_t S = bt->shape[0];
  if (cl->shape[0] != S || (S > 0 && cl->stride[0] != 1)) return PKV_ERR_INVALID_ARG;
  if (!well_formed(qs, 1, PKV_I32) || qs->shape[0] != S + 1 || qs->stride[0] != 1)
    return PKV_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || max_q < 0) return PKV_ERR_INVALID_ARG;
  // q rows are read as 4- (16-bit cache) or 8-byte (fp8 cache) words
  const int qa = fp8 ? 4 : 2;
  if (T > 0 && (q->stride[0] % qa || q->stride[1] % qa || !aligned(q->data, 2 * qa)))
    return PKV_ERR_INVALID_ARG;
  const int64_t g = Hq / Hk;
  if ((D != 64 && D != 128) || (BS != 16 && BS != 32) || (fp8 && D != 128)) return PKV_ERR_UNSUPPORTED;
  if (NB > INT32_MAX || T > INT32_MAX || S * Hk > 65535LL || S > 65535LL ||
      static_cast<int64_t>(max_q) * g > INT32_MAX / 2)
    return PKV_ERR_UNSUPPORTED;
  if (S == 0 || T == 0 || max_q == 0) return PKV_OK;
  if (bt->shape[1] < 1 || NB < 1) return PKV_ERR_INVALID_ARG;
  const int cols = static_cast<int>(max_q * g);
  PrefillLaunch* e = pick_prefill(qdt == PKV_BF16, static_cast<int>(D), BS, cols, fp8);
  if (!e) return PKV_ERR_UNSUPPORTED;
  int dev, st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  DeviceState* ds;
  if ((st = device_state(dev, &ds)) != PKV_OK) return st;
  // 128-row tiles on the tensor cores when a (sequence, head) may have at
  // least 64 rows (a half-filled tile still beats the warp MMAs: 16 new
  // tokens x 4 heads measured 351 us there against 162 us for 32 tokens on
  // the tensor cores), q / out rows are 16-byte aligned (vector loads) and
  // the scale is positive (that kernel takes row maxima of unscaled scores)
  const bool rows16 = q->stride[0] % 8 == 0 && q->stride[1] % 8 == 0 && aligned(q->data, 16) &&
                      out->stride[0] % 8 == 0 && out->stride[1] % 8 == 0 && aligned(out->data, 16);
  // (fp8 caches stay on the warp MMAs: a tcgen05 f16 product takes both
  // operands in one 16-bit type, and these kernels stage K and V as stored)
  const bool use_tc = !fp8 && D == 128 && cols >= 64 && rows16 && scale > 0.f;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!e->attr_set[dev]) {
      if (cudaFuncSetAttribute(e->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, e->smem) !=
          cudaSuccess)
        return PKV_ERR_CUDA;
      e->attr_set[dev] = true;
    }
  }
  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  if ((st = encode_pool_map(&p.tmk, kc, cdt)) != PKV_OK) return st;
  if ((st = encode_pool_map(&p.tmv, vc, cdt)) != PKV_OK) return st;
  p.k_scale = fp8 ? static_cast<const float*>(ks->data) : nullptr;
  p.v_scale = fp8 ? static_cast<const float*>(vs->data) : nullptr;
  p.q = q->data;
  p.q_t = q->stride[0];
  p.q_h = q->stride[1];
  p.out = out->data;
  p.o_t = out->stride[0];
  p.o_h = out->stride[1];
  p.tables = static_cast<const int*>(bt->data);
  p.t_s = bt->stride[0];
  p.lens = static_cast<const int*>(cl->data);
  p.q_start = static_cast<const int*>(qs->data);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.S = static_cast<int>(S);
  p.T = static_cast<int>(T);
  p.Hk = Hk;
  p.g = static_cast<int>(g);
  p.NB = static_cast<int>(NB);
  p.MB = static_cast<int>(bt->shape[1]);
  p.BS = BS;
  if (use_tc) {
    PrefillTcLaunch* te = pick_prefill_tc(qdt == PKV_BF16, BS, static_cast<int>(cols));
    {
      std::lock_guard<std::mutex> lk(g_mu);
      if (!te->attr_set[dev]) {
        if (cudaFuncSetAttribute(te->kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, te->smem) !=
            cudaSuccess)
          return PKV_ERR_CUDA;
        te->attr_set[dev] = true;
      }
    }
    p.err = ds->err;
    p.nkv = 1;
    // longest contexts first, so the last wave of CTAs is short ones (only
    // when there is more than one wave)
    const long long tc_ctas = S * Hk * ((cols + te->rows - 1) / te->rows);
    if (S > 1 && S <= kOrderMaxSeqs && tc_ctas > ds->sms) {
      {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!ds->ord && cudaMalloc(reinterpret_cast<void**>(&ds->ord), kOrderMaxSeqs * sizeof(int)) != cudaSuccess) {
          ds->ord = nullptr;
          return PKV_ERR_CUDA;
        }
      }
      order_by_len_kernel<<<1, kOrderMaxSeqs, 0, stream>>>(p.lens, static_cast<int>(S), ds->ord);
      if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
      p.order = ds->ord;
    }
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t tc = {};
    tc.gridDim = dim3(static_cast<unsigned>((cols + te->rows - 1) / te->rows), 1, static_cast<unsigned>(S * Hk));
    tc.blockDim = dim3(static_cast<unsigned>(te->threads));
    tc.dynamicSmemBytes = static_cast<size_t>(te->smem);
    tc.stream = stream;
    tc.attrs = at;
    tc.numAttrs = 1;
    return cudaLaunchKernelEx(&tc, te->kernel, p) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
  }
  const int ncc = (cols + e->cols - 1) / e->cols;
  p.evict_first = ncc == 1;
  p.err = ds->err;
  p.ccols = e->cols;
  // Few CTAs over long, uneven contexts (short queries): cut each (sequence,
  // head)'s blocks into chunks of 32 (512 or 1024 tokens) so the CTAs are
  // many and even; the partials are merged by a second kernel.
  p.nkv = 1;
  const long long ctas = S * Hk * ncc;
  if (ctas < 4LL * ds->sms && bt->shape[1] > 32) {
    p.kv_chunk = 32;
    p.nkv = static_cast<int>((bt->shape[1] + p.kv_chunk - 1) / p.kv_chunk);
    if (p.nkv > 65535) return PKV_ERR_UNSUPPORTED;
    const size_t rows = static_cast<size_t>(T) * Hq * p.nkv;
    const size_t po = 0, pm = round_up(rows * D * 4, 256), total = round_up(pm + rows * 2 * 4, 256);
    std::lock_guard<std::mutex> lk(g_mu);
    if (ds->pre_bytes < total) {
      if (ds->pre) cudaFree(ds->pre);
      ds->pre = nullptr;
      ds->pre_bytes = 0;
      if (cudaMalloc(&ds->pre, total) != cudaSuccess) return PKV_ERR_CUDA;
      ds->pre_bytes = total;
    }
    p.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(ds->pre) + po);
    p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ds->pre) + pm);
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ncc), static_cast<unsigned>(p.nkv), static_cast<unsigned>(S * Hk));
  cfg.blockDim = dim3(static_cast<unsigned>(e->threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(e->smem);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, e->kernel, p) != cudaSuccess) return PKV_ERR_CUDA;
  if (p.nkv > 1) {
    const long long warps = static_cast<long long>(max_q) * Hq;
    if ((warps + 3) / 4 > INT32_MAX) return PKV_ERR_UNSUPPORTED;
    cfg.gridDim = dim3(static_cast<unsigned>((warps + 3) / 4), static_cast<unsigned>(S));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, e->merge, p) != cudaSuccess) return PKV_ERR_CUDA;
  }
  return PKV_OK;
}

// ---------------------------------------------------------------------------
// Cache writes and block copies
// ---------------------------------------------------------------------------

// Swap blocks between the pools and page-locked host records.
int launch_swap(const pkv_tensor* kc, const pkv_tensor* vc, const pkv_tensor* blocks,
                const void* host, size_t host_bytes, bool out, cudaStream_t stream) {
  if (!kc || !vc || !blocks) return PKV_ERR_INVALID_ARG;
  const int dt = kc->dtype;
  const int eb = elem_bytes(dt);
  if (eb == 0 || eb > 2 || !pool_ok(kc, dt) || !pool_ok(vc, dt) || !same_shape(kc, vc))
    return PKV_ERR_INVALID_ARG;
  if (!well_formed(blocks, 1, PKV_I32)) return PKV_ERR_INVALID_ARG;
  const int64_t n = blocks->shape[0];
  if ((kc->shape[3] * eb) % 16 != 0) return PKV_ERR_UNSUPPORTED;
  if (n > INT32_MAX || kc->shape[0] > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  const long long rec = 2LL * kc->shape[1] * kc->shape[2] * kc->shape[3] * eb;
  if (static_cast<unsigned long long>(n) * rec > host_bytes) return PKV_ERR_INVALID_ARG;
  if (n == 0) return PKV_OK;
  if (!host || !aligned(host, 16)) return PKV_ERR_INVALID_ARG;
  // the host buffer must be page-locked and mapped into the device's space
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, host) != cudaSuccess || at.type != cudaMemoryTypeHost ||
      !at.devicePointer) {
    cudaGetLastError();
    return PKV_ERR_INVALID_ARG;
  }
  int dev, st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  DeviceState* ds;
  if ((st = device_state(dev, &ds)) != PKV_OK) return st;
  SwapParams p;
  std::memset(&p, 0, sizeof(p));
  p.kc = static_cast<uint8_t*>(kc->data);
  p.vc = static_cast<uint8_t*>(vc->data);
  p.c_s0 = kc->stride[0] * eb;
  p.c_s1 = kc->stride[1] * eb;
  p.c_s2 = kc->stride[2] * eb;
  if (vc->stride[0] != kc->stride[0] || vc->stride[1] != kc->stride[1] ||
      vc->stride[2] != kc->stride[2])
    return PKV_ERR_INVALID_ARG;
  p.host = static_cast<uint8_t*>(at.devicePointer);
  p.blocks = static_cast<const int*>(blocks->data);
  p.bl_s = blocks->stride[0];
  p.n = static_cast<int>(n);
  p.Hk = static_cast<int>(kc->shape[1]);
  p.B = static_cast<int>(kc->shape[2]);
  p.NB = static_cast<int>(kc->shape[0]);
  p.row_vecs = static_cast<int>(kc->shape[3] * eb / 16);
  p.rec_bytes = rec;
  const int total = p.Hk * p.B * p.row_vecs;
  const int tpb = 256;
  int chunks = (total + tpb - 1) / tpb;
  if (chunks > 65535) chunks = 65535;
  dim3 grid(static_cast<unsigned>(n), static_cast<unsigned>(chunks));
  if (out)
    swap_blocks_kernel<true><<<grid, tpb, 0, stream>>>(p, ds->err);
  else
    swap_blocks_kernel<false><<<grid, tpb, 0, stream>>>(p, ds->err);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int launch_reshape(const pkv_tensor* k, const pkv_tensor* v, pkv_tensor* kc, pkv_tensor* vc,
                   const pkv_tensor* slots, const pkv_tensor* ks, const pkv_tensor* vs, bool fp8,
                   cudaStream_t stream) {
  if (!k || !v || !kc || !vc || !slots) return PKV_ERR_INVALID_ARG;
  const int xdt = k->dtype;
  if (xdt != PKV_F16 && xdt != PKV_BF16) return PKV_ERR_INVALID_ARG;
  const int cdt = fp8 ? PKV_FP8_E4M3 : xdt;
  if (!well_formed(k, 3, xdt) || !well_formed(v, 3, xdt) || !same_shape(k, v))
    return PKV_ERR_INVALID_ARG;
  if (!pool_ok(kc, cdt) || !pool_ok(vc, cdt) || !same_shape(kc, vc)) return PKV_ERR_INVALID_ARG;
  if (kc->stride[0] != vc->stride[0] || kc->stride[1] != vc->stride[1] ||
      kc->stride[2] != vc->stride[2])
    return PKV_ERR_INVALID_ARG;
  const int64_t T = k->shape[0], Hk = k->shape[1], D = k->shape[2];
  if (kc->shape[1] != Hk || kc->shape[3] != D) return PKV_ERR_INVALID_ARG;
  if (!well_formed(slots, 1, PKV_I64) || slots->shape[0] != T) return PKV_ERR_INVALID_ARG;
  if (T > 0 && slots->stride[0] != 1) return PKV_ERR_INVALID_ARG;
  if (fp8 && (!ks || !vs || !well_formed(ks, 1, PKV_F32) || !well_formed(vs, 1, PKV_F32) ||
              ks->shape[0] != Hk || vs->shape[0] != Hk || ks->stride[0] != 1 ||
              vs->stride[0] != 1))
    return PKV_ERR_INVALID_ARG;
  const int eb = elem_bytes(cdt);
  if ((D * eb) % 16 != 0) return PKV_ERR_UNSUPPORTED;
  // 16-byte vector reads of the inputs
  if (T > 0 && ((k->stride[0] * 2) % 16 || (k->stride[1] * 2) % 16 || (v->stride[0] * 2) % 16 ||
                (v->stride[1] * 2) % 16 || !aligned(k->data, 16) || !aligned(v->data, 16)))
    return PKV_ERR_INVALID_ARG;
  if (T == 0 || Hk == 0) return PKV_OK;
  if (kc->shape[0] > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  int dev, st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  DeviceState* ds;
  if ((st = device_state(dev, &ds)) != PKV_OK) return st;
  CacheParams p;
  std::memset(&p, 0, sizeof(p));
  p.k = static_cast<const uint8_t*>(k->data);
  p.v = static_cast<const uint8_t*>(v->data);
  p.x_s0 = k->stride[0] * 2;
  p.x_s1 = k->stride[1] * 2;
  p.v_s0 = v->stride[0] * 2;
  p.v_s1 = v->stride[1] * 2;
  p.kc = static_cast<uint8_t*>(kc->data);
  p.vc = static_cast<uint8_t*>(vc->data);
  p.c_s0 = kc->stride[0] * eb;
  p.c_s1 = kc->stride[1] * eb;
  p.c_s2 = kc->stride[2] * eb;
  p.slots = static_cast<const long long*>(slots->data);
  p.k_scale = fp8 ? static_cast<const float*>(ks->data) : nullptr;
  p.v_scale = fp8 ? static_cast<const float*>(vs->data) : nullptr;
  p.T = static_cast<int>(T);
  p.Hk = static_cast<int>(Hk);
  p.B = static_cast<int>(kc->shape[2]);
  p.NB = static_cast<int>(kc->shape[0]);
  p.row_vecs = static_cast<int>(D * eb / 16);
  p.in_bytes = static_cast<int>(D * 2);
  const long long threads = T * Hk * p.row_vecs;
  const int tpb = 128;
  const long long blocks = (threads + tpb - 1) / tpb;
  if (blocks > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  void (*kern)(CacheParams, int*) = !fp8                ? reshape_and_cache_kernel
                                    : xdt == PKV_BF16 ? reshape_and_cache_fp8_kernel<true>
                                                      : reshape_and_cache_fp8_kernel<false>;
  return launch_dependent(kern, dim3(static_cast<unsigned>(blocks)), dim3(tpb), stream, p, ds->err);
}

}  // namespace
}  // namespace pkv

// Split-KV scratch of paged_attn_decode_noalloc: a fixed array in device
// memory, created when the library's module is loaded on a device, so that
// call needs no allocation. In host code this name is only a handle: its
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char pkv_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace pkv {
namespace {

void* g_noalloc_ptr[kMaxDevices];

// Device address of pkv_noalloc_scratch on `dev` (which must be current),
// looked up once per device.
int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, pkv_noalloc_scratch);
    if (e != cudaSuccess || !p) return PKV_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return PKV_OK;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

// One new token per sequence (max_q_tokens 1 and as many query rows as
// sequences) is the decode step: the decode kernel serves it (q_start can
// then only be 0, 1, ..., S and is not read). Shapes the decode does not take
// go to the multi-token kernels.
static int prefill_or_decode(const pkv_tensor* q, const pkv_tensor* k_cache,
                             const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                             const pkv_tensor* v_scale, bool fp8, const pkv_tensor* block_tables,
                             const pkv_tensor* context_lens, const pkv_tensor* q_start,
                             int max_q_tokens, int num_kv_heads, float scale, int block_size,
                             pkv_tensor* out, void* stream) {
  if (q && block_tables && max_q_tokens == 1 && q->ndim == 3 && block_tables->ndim == 2 &&
      q->shape[0] == block_tables->shape[0]) {
    DecodeArgs a{q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                 num_kv_heads, scale, block_size, out};
    const int st = launch_decode(a, fp8, nullptr, 0, true, static_cast<cudaStream_t>(stream));
    if (st != PKV_ERR_UNSUPPORTED) return st;
  }
  return launch_prefill(q, k_cache, v_cache, k_scale, v_scale, fp8, block_tables, context_lens,
                        q_start, max_q_tokens, num_kv_heads, scale, block_size, out,
                        static_cast<cudaStream_t>(stream));
}

extern "C" {

const char* pkv_status_string(int s) {
  switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape or type";
    case PKV_ERR_OOM: return "out of free blocks";
    case PKV_ERR_UNKNOWN_SEQ: return "unknown sequence";
    case PKV_ERR_EXISTS: return "sequence exists";
    case PKV_ERR_DOUBLE_FREE: return "double free";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_DEVICE_CHECK: return "device-side check failed";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_SCRATCH_LIMIT: return "request needs more than the static scratch limit";
    default: return "unknown status";
  }
}

int pkv_version(void) { return 100; }

int paged_attn_decode(const pkv_tensor* q, const pkv_tensor* k_cache, const pkv_tensor* v_cache,
                      const pkv_tensor* block_tables, const pkv_tensor* context_lens,
                      int num_kv_heads, float scale, int block_size, pkv_tensor* out,
                      void* stream) {
  DecodeArgs a{q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens,
               num_kv_heads, scale, block_size, out};
  return launch_decode(a, false, nullptr, 0, true, static_cast<cudaStream_t>(stream));
}

int paged_attn_decode_fp8(const pkv_tensor* q, const pkv_tensor* k_cache,
                          const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                          const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                          const pkv_tensor* context_lens, int num_kv_heads, float scale,
                          int block_size, pkv_tensor* out, void* stream) {
  DecodeArgs a{q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
               num_kv_heads, scale, block_size, out};
  return launch_decode(a, true, nullptr, 0, true, static_cast<cudaStream_t>(stream));
}

int paged_attn_decode_cascade(const pkv_tensor* q, const pkv_tensor* k_cache,
                              const pkv_tensor* v_cache, const pkv_tensor* block_tables,
                              const pkv_tensor* context_lens, const pkv_tensor* prefix_blocks,
                              const pkv_tensor* group_start, const pkv_tensor* group_members,
                              int num_groups, int max_group_size, int max_prefix_blocks,
                              int num_kv_heads, float scale, int block_size, pkv_tensor* out,
                              void* stream) {
  DecodeArgs a{q, k_cache, v_cache, nullptr, nullptr, block_tables, context_lens,
               num_kv_heads, scale, block_size, out};
  return launch_cascade(a, false, prefix_blocks, group_start, group_members, num_groups,
                        max_group_size, max_prefix_blocks, static_cast<cudaStream_t>(stream));
}

int paged_attn_decode_cascade_fp8(const pkv_tensor* q, const pkv_tensor* k_cache,
                                  const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                                  const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                                  const pkv_tensor* context_lens, const pkv_tensor* prefix_blocks,
                                  const pkv_tensor* group_start, const pkv_tensor* group_members,
                                  int num_groups, int max_group_size, int max_prefix_blocks,
                                  int num_kv_heads, float scale, int block_size, pkv_tensor* out,
                                  void* stream) {
  DecodeArgs a{q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
               num_kv_heads, scale, block_size, out};
  return launch_cascade(a, true, prefix_blocks, group_start, group_members, num_groups,
                        max_group_size, max_prefix_blocks, static_cast<cudaStream_t>(stream));
}

size_t paged_attn_decode_workspace_bytes(int num_q_heads, int num_kv_heads, int head_dim,
                                         int block_size, int cache_dtype, int device) {
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads || device < 0 || device >= kMaxDevices)
    return 0;
  const bool fp8 = cache_dtype == PKV_FP8_E4M3;
  const int ck = fp8 ? kCacheE4M3 : (cache_dtype == PKV_BF16 ? kCacheBF16 : kCacheF16);
  DecodeLaunch* e = pick_decode(ck, cache_dtype == PKV_BF16 || fp8, head_dim, block_size);
  if (!e) return 0;
  int prev;
  if (cudaGetDevice(&prev) != cudaSuccess) return 0;
  if (prev != device && cudaSetDevice(device) != cudaSuccess) return 0;
  DeviceState* ds;
  int grid = 0;
  size_t bytes = 0;
  if (device_state(device, &ds) == PKV_OK && decode_grid(e, device, ds->sms, &grid) == PKV_OK)
    bytes = ws_default(ds->sms, grid * e->nc, num_q_heads / num_kv_heads, head_dim).total;
  if (prev != device) cudaSetDevice(prev);
  return bytes;
}

int paged_attn_decode_ex(const pkv_tensor* q, const pkv_tensor* k_cache,
                         const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                         const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                         const pkv_tensor* context_lens, int num_kv_heads, float scale,
                         int block_size, pkv_tensor* out, void* workspace,
                         size_t workspace_bytes, unsigned flags, void* stream) {
  if (flags & ~static_cast<unsigned>(PKV_DECODE_DETERMINISTIC)) return PKV_ERR_INVALID_ARG;
  const bool fp8 = k_cache && k_cache->dtype == PKV_FP8_E4M3;
  DecodeArgs a{q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
               num_kv_heads, scale, block_size, out};
  return launch_decode(a, fp8, workspace, workspace_bytes, false,
                       static_cast<cudaStream_t>(stream), false, false, nullptr,
                       (flags & PKV_DECODE_DETERMINISTIC) != 0);
}

// Decode for callers that cannot allocate: the scratch is the static
// pkv_noalloc_scratch array of this file (see the declaration in pagedkv.h).
int paged_attn_decode_noalloc(const pkv_tensor* q, const pkv_tensor* k_cache,
                              const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                              const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                              const pkv_tensor* context_lens, int num_kv_heads, float scale,
                              int block_size, pkv_tensor* out, void* stream) {
  const bool fp8 = k_cache && k_cache->dtype == PKV_FP8_E4M3;
  DecodeArgs a{q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
               num_kv_heads, scale, block_size, out};
  int dev, st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != PKV_OK) return st;
  // launch_decode fits the layout to the array (fewer steal slots when the
  // default does not fit; PKV_ERR_SCRATCH_LIMIT when nothing fits) and, the
  // array keeping the previous call's contents, clears the claim state.
  return launch_decode(a, fp8, scratch, PKV_NOALLOC_SCRATCH_BYTES, false,
                       static_cast<cudaStream_t>(stream), true, true);
}

int reshape_and_cache(const pkv_tensor* k, const pkv_tensor* v, pkv_tensor* k_cache,
                      pkv_tensor* v_cache, const pkv_tensor* slot_mapping, void* stream) {
  return launch_reshape(k, v, k_cache, v_cache, slot_mapping, nullptr, nullptr, false,
                        static_cast<cudaStream_t>(stream));
}

int reshape_and_cache_fp8(const pkv_tensor* k, const pkv_tensor* v, pkv_tensor* k_cache,
                          pkv_tensor* v_cache, const pkv_tensor* slot_mapping,
                          const pkv_tensor* k_scale, const pkv_tensor* v_scale, void* stream) {
  return launch_reshape(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale, true,
                        static_cast<cudaStream_t>(stream));
}

int copy_blocks(pkv_tensor* k_cache, pkv_tensor* v_cache, const pkv_tensor* pairs,
                void* stream) {
  if (!k_cache || !v_cache || !pairs) return PKV_ERR_INVALID_ARG;
  const int dt = k_cache->dtype;
  const int eb = elem_bytes(dt);
  if (eb == 0 || eb > 2 || !pool_ok(k_cache, dt) || !pool_ok(v_cache, dt) ||
      !same_shape(k_cache, v_cache))
    return PKV_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k_cache->stride[i] != v_cache->stride[i]) return PKV_ERR_INVALID_ARG;
  if (!well_formed(pairs, 2, PKV_I32) || pairs->shape[1] != 2) return PKV_ERR_INVALID_ARG;
  const int64_t n = pairs->shape[0];
  if (n == 0) return PKV_OK;
  if ((k_cache->shape[3] * eb) % 16 != 0) return PKV_ERR_UNSUPPORTED;
  if (n > INT32_MAX || k_cache->shape[0] > INT32_MAX) return PKV_ERR_UNSUPPORTED;
  int dev, st;
  if ((st = current_device(&dev)) != PKV_OK) return st;
  DeviceState* ds;
  if ((st = device_state(dev, &ds)) != PKV_OK) return st;
  CopyParams p;
  std::memset(&p, 0, sizeof(p));
  p.kc = static_cast<uint8_t*>(k_cache->data);
  p.vc = static_cast<uint8_t*>(v_cache->data);
  p.c_s0 = k_cache->stride[0] * eb;
  p.c_s1 = k_cache->stride[1] * eb;
  p.c_s2 = k_cache->stride[2] * eb;
  p.pairs = static_cast<const int*>(pairs->data);
  p.pr_s = pairs->stride[0];
  p.n = static_cast<int>(n);
  p.Hk = static_cast<int>(k_cache->shape[1]);
  p.B = static_cast<int>(k_cache->shape[2]);
  p.NB = static_cast<int>(k_cache->shape[0]);
  p.row_vecs = static_cast<int>(k_cache->shape[3] * eb / 16);
  const int total = p.Hk * p.B * p.row_vecs;
  const int tpb = 256;
  int chunks = (total + tpb - 1) / tpb;
  if (chunks > 65535) chunks = 65535;
  dim3 grid(static_cast<unsigned>(n), static_cast<unsigned>(chunks));
  return launch_dependent(copy_blocks_kernel, grid, dim3(tpb), static_cast<cudaStream_t>(stream), p, ds->err);
}


int paged_attn_prefill(const pkv_tensor* q, const pkv_tensor* k_cache, const pkv_tensor* v_cache,
                       const pkv_tensor* block_tables, const pkv_tensor* context_lens,
                       const pkv_tensor* q_start, int max_q_tokens, int num_kv_heads, float scale,
                       int block_size, pkv_tensor* out, void* stream) {
  return prefill_or_decode(q, k_cache, v_cache, nullptr, nullptr, false, block_tables, context_lens,
                           q_start, max_q_tokens, num_kv_heads, scale, block_size, out, stream);
}

int paged_attn_prefill_fp8(const pkv_tensor* q, const pkv_tensor* k_cache,
                           const pkv_tensor* v_cache, const pkv_tensor* k_scale,
                           const pkv_tensor* v_scale, const pkv_tensor* block_tables,
                           const pkv_tensor* context_lens, const pkv_tensor* q_start,
                           int max_q_tokens, int num_kv_heads, float scale, int block_size,
                           pkv_tensor* out, void* stream) {
  return prefill_or_decode(q, k_cache, v_cache, k_scale, v_scale, true, block_tables, context_lens,
                           q_start, max_q_tokens, num_kv_heads, scale, block_size, out, stream);
}

int swap_out_blocks(const pkv_tensor* k_cache, const pkv_tensor* v_cache, const pkv_tensor* blocks,
                    void* host_dst, size_t host_bytes, void* stream) {
  return launch_swap(k_cache, v_cache, blocks, host_dst, host_bytes, true,
                     static_cast<cudaStream_t>(stream));
}

int swap_in_blocks(const void* host_src, size_t host_bytes, const pkv_tensor* blocks,
                   pkv_tensor* k_cache, pkv_tensor* v_cache, void* stream) {
  return launch_swap(k_cache, v_cache, blocks, host_src, host_bytes, false,
                     static_cast<cudaStream_t>(stream));
}

int pkv_device_error(int device) {
  if (device < 0 || device >= kMaxDevices) return PKV_ERR_INVALID_ARG;
  int prev;
  if (cudaGetDevice(&prev) != cudaSuccess) return PKV_ERR_CUDA;
  if (prev != device && cudaSetDevice(device) != cudaSuccess) return PKV_ERR_CUDA;
  int st = PKV_OK;
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpyFromSymbol(&v, g_pkv_err, sizeof(int)) != cudaSuccess) {
    st = PKV_ERR_CUDA;
  } else if (v != 0) {
    const int zero = 0;
    st = cudaMemcpyToSymbol(g_pkv_err, &zero, sizeof(int)) == cudaSuccess ? PKV_ERR_DEVICE_CHECK
                                                                           : PKV_ERR_CUDA;
  }
  if (prev != device) cudaSetDevice(prev);
  return st;
}

}  // extern "C"
