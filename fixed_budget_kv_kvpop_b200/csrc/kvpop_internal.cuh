// Internal definitions shared by the KVpop CUDA kernels and the C-ABI host code.
//
// Method: "KVpop -- Key-Value Cache Compression with Predictive Online Pruning"
// (summary page of arXiv 2607.05061v2).  Each KV head keeps a bounded cache of
// S sink tokens, a protected window of the W most recent tokens, an optional
// D-slot staging ring for delayed scoring, and K long-range slots holding the
// running top-k of the tokens that have left the window (§3 Fixed-budget
// pruning, §C.1 Mask Definition, §I Pseudocode).
//
// Device cache layout of one layer (all row-major, one "unit" = one
// (batch row, KV head) pair, unit = b * Hkv + h):
//   kv    [units][NS][2][d]  element type T; per slot the key row then the value
//                            row, so one slot is one contiguous 2*d*sizeof(T) row
//   pos   [units][NS]  int32 position held by each slot, -1 = empty
//   score [units][NS]  fp32  ranking score (long-range slots; with caller
//                            scores also the window/staging slots)
//   state [units][4]   int32 {n_seen, n_topk, 0, 0} (per unit, for inspection)
//   layer  LayerState  {n_seen, n_topk, ticket}: the counters every kernel of
//                      the layer reads; updated only by the last warp of a
//                      launch, so all warps of a launch see the same values
//   dec   [2][units]   Decision: the eviction decision of the step appending
//                      token N lives in dec[N & 1] (taken one step ahead)
// Slot map: sinks [0, S) hold positions 0..S-1; window slot of token t is
// S + (t mod W); staging slot is S + W + (t mod D); long-range slots start at
// S + W + D and fill as a prefix.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace kvpop {

// Device error bits, OR-ed into the error word (read by kvpop_get_error).
enum : int32_t {
  DEVERR_CONTEXT_OVERFLOW = 1,
  DEVERR_TIMEOUT = 2,
  DEVERR_BAD_INDEX = 4,
  DEVERR_NAN_SCORE = 8,
  DEVERR_STATE_MISMATCH = 16,
};

constexpr int kMaxSeg = 64;         // split-K partials per unit (upper bound)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded mbarrier waits: 2 s
// Bound of the decode kernel's merge-queue waits (shared memory only, no copy
// in flight).  Test builds shorten it to make such a wait run out quickly.
#ifndef KVPOP_MERGE_WAIT_LIMIT_NS
#define KVPOP_MERGE_WAIT_LIMIT_NS 2000000000ull
#endif
constexpr uint64_t kMergeWaitLimitNs = KVPOP_MERGE_WAIT_LIMIT_NS;

// Per-layer counters shared by all units (all batch rows share one length).
struct LayerState {
  int32_t n_seen;   // tokens in the cache; the next decode step appends token n_seen
  int32_t n_topk;   // long-range slots in use (a prefix of the long-range region)
  int32_t ticket;   // warps of the current launch that have finished
  int32_t pad;
};

// Eviction decision of the decode step that appends token p, for one unit.
// The token b = p - W - D reaches the eviction boundary at that step.
struct Decision {
  int32_t p;       // position the decision is for
  int32_t bpos;    // boundary token position, -1 if none
  int32_t bslot;   // its slot before the step's moves
  int32_t tgt;     // long-range slot it moves to, -1 if dropped (or none)
  int32_t evict;   // slot whose token leaves the attended set at this step, -1 if none
  float sb;        // its ranking score
  int32_t pad[2];
};

struct LayerArgs {
  uint8_t* kv;          // this layer's [units][NS][2][d]
  int32_t* pos;         // [units][NS]
  float* score;         // [units][NS]
  int32_t* state;       // [units][4]
  LayerState* layer;    // this layer's counters
  Decision* dec;        // [2][units]
  const float* w1;      // this layer's scorer [Hkv][hidden][2d]
  const float* b1;      // [Hkv][hidden]
  const float* w2;      // [Hkv][hidden]
  const float* b2;      // [Hkv]
  int32_t* err;         // device error word
  int units, Hkv, Hq, G, d, S, W, D, K, NS, hidden;
  int max_context;
  uint32_t flags;
  int row_bytes;        // 2 * d * sizeof(T)
  const float* log_decay;   // this layer's ln(gamma) [Hkv], or null (no temporal decay)
  // Stateful mLSTM scorer (page §A, §E.3, §E.4); mlstm = 0 when the stateless
  // scorer or caller scores decide.
  int mlstm;            // 1: each step's decision waits for the step's own token
  int mp, mdv;          // Hedgehog projection size p (2p features), value size dv
  const float* mw;      // this layer's weights [Hkv][mlstm_head_floats(p, dv, d)]
  double* mstate;       // this layer's states [units][mlstm_state_doubles(p, dv)]
  int test_hook;        // failure injection, honoured only by builds with KVPOP_TEST_HOOKS
};

// test_hook values (KVPOP_TEST_HOOKS builds): consumer warp 0 of CTA 0 does
// its work but never reports that it is done, so the CTA's merge helpers wait
// until kMergeWaitLimitNs and record DEVERR_TIMEOUT.
constexpr int TEST_HOOK_WITHHOLD_DONE = 1;

// mLSTM weights of one (layer, KV head): rows of 2d floats W_q [p], W_k [p],
// W_v [dv], w_i, w_f; then w_o [dv], b_i, b_f, b_o, padded to 4 floats.
__host__ __device__ __forceinline__ int mlstm_head_floats(int p, int dv, int d) {
  return (2 * p + dv + 2) * 2 * d + ((dv + 3 + 3) / 4) * 4;
}
// State of one unit, fp64: C [2p][dv] (feature-major), n [2p], m, pad.
__host__ __device__ __forceinline__ int mlstm_state_doubles(int p, int dv) { return 2 * p * dv + 2 * p + 2; }

// Scorer weights of KV head h in this layer: W1 rows (one row for the linear
// scorer), b1 and w2 (null for the linear scorer).
__host__ __device__ __forceinline__ const float* head_w1(const LayerArgs& a, int h) {
  return a.w1 + static_cast<size_t>(h) * (a.hidden > 0 ? a.hidden : 1) * 2 * a.d;
}
__host__ __device__ __forceinline__ const float* head_b1(const LayerArgs& a, int h) {
  return a.hidden > 0 ? a.b1 + static_cast<size_t>(h) * a.hidden : nullptr;
}
__host__ __device__ __forceinline__ const float* head_w2(const LayerArgs& a, int h) {
  return a.hidden > 0 ? a.w2 + static_cast<size_t>(h) * a.hidden : nullptr;
}

// Ranking priority of a token that becomes eligible at step e: its score, or
// with temporal decay the static priority s - e * ln(gamma_h) in one fp32
// rounding (page §B.3; e <= 2^24 is exact in fp32).
__device__ __forceinline__ float ranking_priority(const LayerArgs& a, int unit, int e, float s) {
  if (a.log_decay == nullptr) return s;
  return __fmaf_rn(-static_cast<float>(e), a.log_decay[unit % a.Hkv], s);
}

constexpr uint32_t FLAG_EXTERNAL_SCORES = 1u;
constexpr uint32_t FLAG_DEBUG_CHECKS = 2u;

// --- total order on tokens: key = (score, -position), packed in 64 bits ---
// Higher score ranks higher; on equal score the older (smaller) position ranks
// higher.  -0.0 is folded onto +0.0 and NaN ranks below -inf.
__host__ __device__ __forceinline__ uint64_t rank_key(float s, int32_t pos) {
  uint32_t u;
#ifdef __CUDA_ARCH__
  u = __float_as_uint(s);
#else
  __builtin_memcpy(&u, &s, 4);
#endif
  uint32_t ordered;
  if ((u & 0x7fffffffu) > 0x7f800000u) {
    ordered = 0u;                       // NaN
  } else {
    if ((u & 0x7fffffffu) == 0u) u = 0u;  // -0 -> +0
    ordered = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  }
  return (static_cast<uint64_t>(ordered) << 32) | static_cast<uint32_t>(0xffffffffu - static_cast<uint32_t>(pos));
}

// --- slot helpers ---
__host__ __device__ __forceinline__ int window_slot(int t, int S, int W) { return S + (t % W); }
__host__ __device__ __forceinline__ int staging_slot(int t, int S, int W, int D) { return S + W + (t % D); }
__host__ __device__ __forceinline__ int topk_base(int S, int W, int D) { return S + W + D; }

// Split-K work decomposition of the decode kernel (host and device agree on it).
// total tiles = units * tpu; nw = number of consumer warps that get work; warp
// w covers tiles [w*total/nw, (w+1)*total/nw).
__host__ __device__ __forceinline__ int64_t seg_lo(int64_t w, int64_t total, int64_t nw) {
  return (w * total) / nw;
}
__host__ __device__ __forceinline__ int64_t warp_of_tile(int64_t x, int64_t total, int64_t nw) {
  return ((x + 1) * nw - 1) / total;
}
__host__ __device__ __forceinline__ int64_t decode_active_warps(int64_t total, int64_t tpu, int64_t launched) {
  int64_t nw = launched < total ? launched : total;
  // every unit must be covered by at most kMaxSeg warps
  int64_t min_tiles = (tpu + (kMaxSeg - 2)) / (kMaxSeg - 1);
  if (min_tiles < 1) min_tiles = 1;
  int64_t cap = total / min_tiles;
  if (cap < 1) cap = 1;
  return nw < cap ? nw : cap;
}


// --- element conversions ---
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float x) { return x; }
  static __device__ __forceinline__ float from_f32(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// Unpack 16 bytes (one uint4) into fp32 values.
__device__ __forceinline__ void unpack16(const uint4& r, float* out, float) {
  out[0] = __uint_as_float(r.x); out[1] = __uint_as_float(r.y);
  out[2] = __uint_as_float(r.z); out[3] = __uint_as_float(r.w);
}
__device__ __forceinline__ void unpack16(const uint4& r, float* out, __nv_bfloat16) {
  out[0] = __uint_as_float(r.x << 16); out[1] = __uint_as_float(r.x & 0xffff0000u);
  out[2] = __uint_as_float(r.y << 16); out[3] = __uint_as_float(r.y & 0xffff0000u);
  out[4] = __uint_as_float(r.z << 16); out[5] = __uint_as_float(r.z & 0xffff0000u);
  out[6] = __uint_as_float(r.w << 16); out[7] = __uint_as_float(r.w & 0xffff0000u);
}

// --- mbarrier / bulk-copy wrappers (sm_90+ PTX, used here on sm_100a) ---
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait: returns false (and the caller records DEVERR_TIMEOUT) when the
// phase does not complete within kWaitLimitNs of wall time.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}
// One contiguous global -> shared bulk copy (no multicast), completion counted
// in bytes on the mbarrier.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// L2 prefetch of one contiguous range (a hint: no data moves to the SM and
// nothing waits).  addr and bytes must be multiples of 16.
__device__ __forceinline__ void prefetch_l2(const void* addr, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(addr), "r"(bytes) : "memory");
}

__device__ __forceinline__ int ld_relaxed(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void set_error(int32_t* err, int32_t bits) {
  atomicOr(err, bits);
}

// Scorer: s = w2 . relu(W1 x + b1) + b2 for x = [k; v] of one token (KVpop
// page §E.1 headwise inputs, §E.2 stateless MLP scorer), computed by one warp.
// Accumulated in fp64 (bf16/fp32 inputs and fp32 weights are exact in fp64)
// and rounded once to fp32, the ranking precision (§F).  Lane l holds inputs
// [l * X, l * X + X) of [k; v] (X = 2d / 32) in fp64; for each hidden row the
// warp reads the whole W1 row (coalesced: 4 cache lines per instruction), each
// lane forms its X-term partial sum, and a butterfly reduction over 16 rows at
// a time leaves lane l (< 16) with the pre-activation of row 16 * block + l.
// Lane l of a warp loads inputs [l X, l X + X) of x = [k; v] (X = D2 / 32) as
// fp64 (bf16 / fp32 inputs are exact in fp64).  krow, vrow 16-byte aligned.
template <typename T, int D2>
__device__ __forceinline__ void load_scorer_input(const T* krow, const T* vrow, double (&x)[D2 / 32]) {
  constexpr int X = D2 / 32;      // inputs per lane (4 or 8)
  constexpr int D = D2 / 2;
  const int lane = threadIdx.x & 31;
  const int i0 = lane * X;
  const T* src = (i0 < D) ? krow + i0 : vrow + (i0 - D);
  constexpr int kBytes = X * static_cast<int>(sizeof(T));   // 8, 16 or 32: rows are 16-byte aligned
  alignas(16) T xr[X];
  if constexpr (kBytes % 16 == 0) {
#pragma unroll
    for (int q = 0; q < kBytes / 16; ++q) reinterpret_cast<uint4*>(xr)[q] = reinterpret_cast<const uint4*>(src)[q];
  } else {
    reinterpret_cast<uint2*>(xr)[0] = reinterpret_cast<const uint2*>(src)[0];
  }
#pragma unroll
  for (int e = 0; e < X; ++e) x[e] = static_cast<double>(Elem<T>::to_f32(xr[e]));
}

// Scorer: s = w2 . relu(W1 x + b1) + b2 for x = [k; v] of one token (KVpop
// page §E.1 headwise inputs, §E.2 stateless MLP scorer), computed by one warp
// from the inputs load_scorer_input placed in its lanes.  Accumulated in fp64
// and rounded once to fp32, the ranking precision (§F).  For each hidden row
// the warp reads the whole W1 row (coalesced: 4 cache lines per instruction),
// each lane forms its X-term partial sum, and a butterfly reduction over 16
// rows at a time leaves lane l (< 16) with the pre-activation of row
// 16 * block + l.  mlp_part_x sums w2_j relu(.) over the hidden rows
// [j0, j1) (whole blocks of 16) and returns it in every lane, without b2.
template <int D2, int HID>
__device__ __forceinline__ double mlp_part_x(const double (&x)[D2 / 32], const float* w1, const float* b1,
                                             const float* w2, int j0, int j1) {
  constexpr int X = D2 / 32;
  const int lane = threadIdx.x & 31;
  const int i0 = lane * X;
  double part = 0.0;
  for (int blk = j0; blk < j1; blk += 16) {
    // b1 and w2 of the row this lane finishes, issued with the block's W1 loads
    const float b1j = (lane < 16) ? __ldg(b1 + blk + lane) : 0.f;
    const float w2j = (lane < 16) ? __ldg(w2 + blk + lane) : 0.f;
    double v[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const float4* wr = reinterpret_cast<const float4*>(w1 + static_cast<size_t>(blk + r) * D2 + i0);
      double acc = 0.0;
#pragma unroll
      for (int q = 0; q < X / 4; ++q) {
        const float4 w = __ldg(wr + q);
        acc = fma(static_cast<double>(w.x), x[4 * q + 0], acc);
        acc = fma(static_cast<double>(w.y), x[4 * q + 1], acc);
        acc = fma(static_cast<double>(w.z), x[4 * q + 2], acc);
        acc = fma(static_cast<double>(w.w), x[4 * q + 3], acc);
      }
      v[r] = acc;
    }
    // fold the two half-warps, then reduce-scatter over the 16 lanes of each:
    // after the step with offset o, lane l keeps the half of its values whose
    // index has bit o equal to l's; lanes l and l ^ 16 end with row l & 15
#pragma unroll
    for (int r = 0; r < 16; ++r) v[r] += __shfl_xor_sync(0xffffffffu, v[r], 16);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const double keep = up ? v[i + o] : v[i];
        const double send = up ? v[i] : v[i + o];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    if (lane < 16) part = fma(static_cast<double>(w2j), fmax(v[0] + static_cast<double>(b1j), 0.0), part);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  return part;
}

template <int D2, int HID>
__device__ __forceinline__ float mlp_score_x(const double (&x)[D2 / 32], const float* w1, const float* b1,
                                             const float* w2, float b2) {
  return static_cast<float>(mlp_part_x<D2, HID>(x, w1, b1, w2, 0, HID) + static_cast<double>(b2));
}

template <typename T, int D2, int HID>
__device__ __forceinline__ float mlp_score_rows(const T* krow, const T* vrow, const float* w1, const float* b1,
                                                const float* w2, float b2) {
  double x[D2 / 32];
  load_scorer_input<T, D2>(krow, vrow, x);
  return mlp_score_x<D2, HID>(x, w1, b1, w2, b2);
}

// Stateless headwise linear scorer s = w . [k; v] + b (page §E.2), one warp:
// lane l holds inputs [l * X, l * X + X) and the matching weights; fp64 dot
// product, warp reduction, one rounding to fp32.
template <int D2>
__device__ __forceinline__ float linear_score_x(const double (&x)[D2 / 32], const float* w, float b) {
  constexpr int X = D2 / 32;
  const int i0 = (threadIdx.x & 31) * X;
  double acc = 0.0;
#pragma unroll
  for (int q = 0; q < X / 4; ++q) {
    const float4 wv = __ldg(reinterpret_cast<const float4*>(w + i0) + q);
    acc = fma(static_cast<double>(wv.x), x[4 * q + 0], acc);
    acc = fma(static_cast<double>(wv.y), x[4 * q + 1], acc);
    acc = fma(static_cast<double>(wv.z), x[4 * q + 2], acc);
    acc = fma(static_cast<double>(wv.w), x[4 * q + 3], acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return static_cast<float>(acc + static_cast<double>(b));
}

template <typename T, int D2>
__device__ __forceinline__ float linear_score_rows(const T* krow, const T* vrow, const float* w, float b) {
  double x[D2 / 32];
  load_scorer_input<T, D2>(krow, vrow, x);
  return linear_score_x<D2>(x, w, b);
}

// hidden in {32, 64, 128} (MLP) or 0 (linear: w1 is the weight row, b2 the
// bias); d = 64 or 128; krow, vrow 16-byte aligned.  Returns the score in
// every lane.
template <typename T>
__device__ __noinline__ float mlp_score_warp(const T* krow, const T* vrow, int d, const float* w1, const float* b1,
                                             const float* w2, float b2, int hidden) {
  if (hidden == 0) {
    if (d == 128) return linear_score_rows<T, 256>(krow, vrow, w1, b2);
    return linear_score_rows<T, 128>(krow, vrow, w1, b2);
  }
  if (d == 128) {
    if (hidden == 32) return mlp_score_rows<T, 256, 32>(krow, vrow, w1, b1, w2, b2);
    if (hidden == 64) return mlp_score_rows<T, 256, 64>(krow, vrow, w1, b1, w2, b2);
    return mlp_score_rows<T, 256, 128>(krow, vrow, w1, b1, w2, b2);
  }
  if (hidden == 32) return mlp_score_rows<T, 128, 32>(krow, vrow, w1, b1, w2, b2);
  if (hidden == 64) return mlp_score_rows<T, 128, 64>(krow, vrow, w1, b1, w2, b2);
  return mlp_score_rows<T, 128, 128>(krow, vrow, w1, b1, w2, b2);
}

// Minimum key (score, -position) of the long-range slots base + [i_lo, i_hi)
// (pending's target counting with pending's key), in every lane of the warp;
// ~0 and slot -1 for an empty range.
__device__ __forceinline__ uint64_t longrange_min(const LayerArgs& a, int u, const Decision* pending, int i_lo,
                                                  int i_hi, int& mslot) {
  const int lane = threadIdx.x & 31;
  const int base = topk_base(a.S, a.W, a.D);
  const int32_t* pos = a.pos + static_cast<size_t>(u) * a.NS;
  const float* score = a.score + static_cast<size_t>(u) * a.NS;
  constexpr int kB = 16;   // long-range keys per lane per round trip
  uint64_t best = ~0ull;
  mslot = -1;
  for (int i0 = i_lo; i0 < i_hi; i0 += 32 * kB) {
    float sc[kB];
    int32_t ps[kB];
#pragma unroll
    for (int t = 0; t < kB; ++t) {
      const int i = i0 + lane + 32 * t;
      if (i < i_hi) { sc[t] = score[base + i]; ps[t] = pos[base + i]; }
    }
#pragma unroll
    for (int t = 0; t < kB; ++t) {
      const int i = i0 + lane + 32 * t;
      if (i < i_hi) {
        const int sl = base + i;
        const uint64_t key = (pending != nullptr && sl == pending->tgt) ? rank_key(pending->sb, pending->bpos)
                                                                        : rank_key(sc[t], ps[t]);
        if (key < best) { best = key; mslot = sl; }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t ok = __shfl_xor_sync(0xffffffffu, best, o);
    const int os = __shfl_xor_sync(0xffffffffu, mslot, o);
    if (ok < best) { best = ok; mslot = os; }
  }
  return best;
}

// Eviction decision against the long-range set, taken by one warp for the
// boundary token b (ranking priority sb) of unit u; r.bslot is set.  While
// fewer than K long-range slots are used (ntk < K), b takes the next free
// one.  Otherwise the warp finds the minimum key (score, -position) of the
// long-range slots and b replaces it only if its own key is strictly larger;
// else b is dropped.  pending: the previous step's decision when it is not
// yet committed (its target slot then counts with pending's key), or null.
// Keys are unique (positions are), so the argmin is unique.
__device__ __forceinline__ void longrange_decide(const LayerArgs& a, int u, int ntk, const Decision* pending,
                                                 float sb, int b, Decision& r) {
  const int K = a.K;
  const int base = topk_base(a.S, a.W, a.D);
  if (ntk < K) {
    r.tgt = base + ntk;     // fill-up: next free long-range slot, nobody leaves
    r.evict = -1;
    return;
  }
  if (K == 0) {
    r.evict = r.bslot;
    return;
  }
  int mslot;
  const uint64_t best = longrange_min(a, u, pending, 0, K, mslot);
  if (rank_key(sb, b) > best) {
    r.tgt = mslot;
    r.evict = mslot;
  } else {
    r.evict = r.bslot;
  }
}

// Packed fp32 FMA (sm_100 FFMA2): d = a * b + c on both halves, round-to-nearest.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// bf16x2 word -> (lo, hi) as fp32 (exact).
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Warp-level bf16 tensor-core helpers (mma.sync m16n8k16, fp32 accumulate)
// and the shared-memory matrix loads that feed them.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t* r) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
               "{%8, %9}, {%0, %1, %2, %3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// (lo, hi) -> bf16x2 word, round to nearest even; lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Decode kernel scratch (split-K partials), shared by the layers of a handle.
struct DecodeScratch {
  float* part_acc;    // [units][kMaxSeg][G][d]
  float* part_ml;     // [units][kMaxSeg][G][2]
  int32_t* ticket;    // [units]
};

// Kernel launchers (defined in the .cu files).
enum DecodeMode : int { MODE_STEP = 0, MODE_ATTEND = 1, MODE_STEP_NODECIDE = 2 };
// One fused decode step (MODE_STEP), the same step taking its decision from a
// kernel launched just before it instead of deciding the next step
// (MODE_STEP_NODECIDE, the mLSTM scorer), or attention over the cache as it
// stands (MODE_ATTEND).  ext_score may be null.
int launch_decode(const CUtensorMap& tmap, const LayerArgs& a, int dtype, const DecodeScratch& sc, int mode,
                  const void* q, const void* k_new, const void* v_new, const float* ext_score, void* out, int num_sms,
                  cudaStream_t st);
// Tensor map over one layer's cache rows for the decode kernel's TMA loads.
int make_decode_tensor_map(CUtensorMap* map, void* layer_kv, int dtype, int d, int64_t rows, int row_bytes);
// The cache update of a decode step without attention.
int launch_append(const LayerArgs& a, int dtype, const void* k_new, const void* v_new, const float* ext_score,
                  cudaStream_t st);
// Takes the eviction decision for the next decode step from the cache as it
// stands and sets the layer counters to (n_seen, n_topk).
int launch_decide(const LayerArgs& a, int dtype, int n_seen, int n_topk, cudaStream_t st);
int decode_supported(int dtype, int d, int G);

struct PrefillScratch {
  float* new_score;   // [units][cap]
  int32_t* tgt;       // [units][K]
  int cap;            // capacity of newly eligible tokens per unit per chunk
};
int launch_prefill(const LayerArgs& a, int dtype, const PrefillScratch& ps, const void* k, const void* v,
                   int n_tokens, int n_seen_before, int n_topk_before, const float* ext_scores,
                   cudaStream_t st);

// mLSTM scorer (kvpop_mlstm.cu).  Decode: updates every unit's state with the
// step's token and writes the step's eviction decision (dec[N & 1]) for the
// decode kernel that follows in MODE_STEP_NODECIDE.  Prefill: runs the
// recurrence over the chunk of tokens [n0, n0 + n) and writes the ranking
// priority of every token that becomes eligible in it into
// out[u * cap + (t - e0)].  Both return 0 or -1 (launch failed).
int launch_mlstm_step(const LayerArgs& a, int dtype, const void* k_new, const void* v_new, cudaStream_t st);
int launch_mlstm_prefill(const LayerArgs& a, int dtype, const void* k, const void* v, int n, int n0, int e0,
                         float* out, int cap, cudaStream_t st);

}  // namespace kvpop
