// Stateful mLSTM scorer with delayed readout (KVpop page §A "Background:
// Linear Attention and mLSTM", §E.3 "mLSTM Scorer", §E.4 "Delayed Readout").
//
// Per KV head a recurrent state in fp64: matrix memory C [2p][dv] (stored
// feature-major: lane f of a warp owns row f), normaliser n [2p] and the
// stabiliser m.  Every token t with x_t = [k_t; v_t] (§E.1) updates it:
//   phi   = [softmax(z); softmax(-z)],  z = W_k x_t      (Hedgehog, 2p features)
//   i~    = w_i . x_t + b_i,   log f = log sigmoid(w_f . x_t + b_f)
//   m'    = max(log f + m, i~),  i' = exp(i~ - m'),  f' = exp(log f + m - m')
//   C'    = f' C + i' phi (W_v x_t)^T,   n' = f' n + i' phi
// (the stabilised form of the gated outer-product sum; no output gate).  The
// token u that becomes eligible at step q = u + W + D is read out from the
// state after token q, with read features r = Hedgehog(W_q x_u):
//   h = C^T r / max(|n . r|, exp(-m)),   score = w_o . SiLU(h) + b_o,
// rounded once to fp32, the ranking precision (§F).
//
// One warp per (batch row, KV head) unit.  Lane l holds inputs
// [l X, l X + X) of x (X = 2d / 32) in fp64; a projection onto up to 32 rows
// is a per-lane partial dot product per row followed by a warp sum that lane
// j keeps for row j (a rolled loop: the step kernel runs from a cold
// instruction cache after every decode kernel, so its code is kept short).  Weights are fp32 and inputs bf16 or fp32, both
// exact in fp64.
//
// Decode: mlstm_step_kernel (one CTA of four warps per unit, the head's
// projection weights staged in shared memory) runs before each decode
// kernel of a layer.  It folds the step's token into the state and
// takes that step's eviction decision (the boundary token's score depends on the token that arrives in
// the same step, so the decision cannot be taken one step ahead as the
// stateless scorers' is).  Prefill: mlstm_prefill_kernel walks a chunk's
// tokens in order and scores each token as it becomes eligible.
#include "kvpop_internal.cuh"

namespace kvpop {

namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMlstmWarps = 4;   // units per block

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Lane l loads inputs [l X, l X + X) of x = [k; v] as fp64 (d = 16 X).
template <typename T, int X>
__device__ __forceinline__ void load_x(const T* krow, const T* vrow, double (&x)[X]) {
  constexpr int D = 16 * X;
  const int i0 = (threadIdx.x & 31) * X;
  const T* src = (i0 < D) ? krow + i0 : vrow + (i0 - D);
  constexpr int kBytes = X * static_cast<int>(sizeof(T));   // 8, 16 or 32; rows are 16-byte aligned
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

// Dot products of x with rows [r0, r0 + nr) (nr <= 32) of a row-major fp32
// matrix with 32 X columns; row r0 + j ends in lane j (0 in lanes >= nr).
// kShared: w is in shared memory (plain loads), else global (read-only loads).
template <int X, bool kShared = false>
__device__ __forceinline__ double project_rows(const double (&x)[X], const float* __restrict__ w, int r0, int nr) {
  const int lane = threadIdx.x & 31;
  double out = 0.0;
#pragma unroll 1
  for (int r = 0; r < nr; ++r) {
    const float4* wr = reinterpret_cast<const float4*>(w + static_cast<size_t>(r0 + r) * (32 * X) + lane * X);
    double acc = 0.0;
#pragma unroll
    for (int q = 0; q < X / 4; ++q) {
      float4 c;
      if constexpr (kShared) c = wr[q];
      else c = __ldg(wr + q);
      acc = fma(static_cast<double>(c.x), x[4 * q + 0], acc);
      acc = fma(static_cast<double>(c.y), x[4 * q + 1], acc);
      acc = fma(static_cast<double>(c.z), x[4 * q + 2], acc);
      acc = fma(static_cast<double>(c.w), x[4 * q + 3], acc);
    }
    acc = warp_sum(acc);
    if (lane == r) out = acc;
  }
  return out;
}

// Hedgehog features of z (z_j in lane j < p): [softmax(z); softmax(-z)],
// feature f in lane f < 2p, 0 in the other lanes.
__device__ __forceinline__ double hedgehog_lane(double z, int p) {
  const int lane = threadIdx.x & 31;
  const double mp = warp_max(lane < p ? z : -__builtin_huge_val());
  const double mn = warp_max(lane < p ? -z : -__builtin_huge_val());
  const double zz = __shfl_sync(kFull, z, lane < p ? lane : lane - p);
  const bool pos = lane < p, neg = lane >= p && lane < 2 * p;
  double e = 0.0;
  if (pos) e = exp(zz - mp);
  else if (neg) e = exp(-zz - mn);
  const double sp = warp_sum(pos ? e : 0.0);
  const double sn = warp_sum(neg ? e : 0.0);
  return pos ? e / sp : (neg ? e / sn : 0.0);
}

__device__ __forceinline__ double log_sigmoid(double x) {
  return x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x));
}

// Per-lane view of one unit's state: lane f < 2p holds C[f][0..dv) and n[f];
// m in every lane.
template <int DV>
struct LaneState {
  double c[DV];
  double n;
  double m;
};

template <int DV>
__device__ __forceinline__ void state_load(const double* st, int p, int dv, LaneState<DV>& s) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < DV; ++j) s.c[j] = (lane < 2 * p && j < dv) ? st[lane * dv + j] : 0.0;
  s.n = lane < 2 * p ? st[2 * p * dv + lane] : 0.0;
  s.m = st[2 * p * dv + 2 * p];
}
template <int DV>
__device__ __forceinline__ void state_store(double* st, int p, int dv, const LaneState<DV>& s) {
  const int lane = threadIdx.x & 31;
  if (lane < 2 * p) {
#pragma unroll
    for (int j = 0; j < DV; ++j)
      if (j < dv) st[lane * dv + j] = s.c[j];
    st[2 * p * dv + lane] = s.n;
  }
  if (lane == 0) st[2 * p * dv + 2 * p] = s.m;
}

// Folds token x into the state (weights hw of the unit's KV head).
template <int X, int DV>
__device__ __forceinline__ void state_update(const double (&x)[X], const float* __restrict__ hw, int p, int dv,
                                             LaneState<DV>& s) {
  const int R = 2 * p + dv + 2;
  const float* tail = hw + static_cast<size_t>(R) * (32 * X);
  const double phi = hedgehog_lane(project_rows<X>(x, hw, p, p), p);
  const double val = project_rows<X>(x, hw, 2 * p, dv);
  const double g = project_rows<X>(x, hw, 2 * p + dv, 2);
  const double gi = __shfl_sync(kFull, g, 0) + static_cast<double>(__ldg(tail + dv));
  const double gf = __shfl_sync(kFull, g, 1) + static_cast<double>(__ldg(tail + dv + 1));
  const double lf = log_sigmoid(gf);
  const double m_new = fmax(lf + s.m, gi);
  const double ip = exp(gi - m_new);
  const double fp = exp(lf + s.m - m_new);
#pragma unroll
  for (int j = 0; j < DV; ++j) {
    const double vj = __shfl_sync(kFull, val, j);
    if (j < dv) s.c[j] = fp * s.c[j] + ip * (vj * phi);
  }
  s.n = fp * s.n + ip * phi;
  s.m = m_new;
}

// Delayed readout from the state of a token with read features r (feature f
// in lane f): h = C^T r / max(|n . r|, e^-m), score = w_o . SiLU(h) + b_o,
// rounded once to fp32 (tail: w_o, b_i, b_f, b_o of the head).
template <int DV>
__device__ __forceinline__ float state_readout(double r, const float* __restrict__ tail, int dv,
                                               const LaneState<DV>& s) {
  const int lane = threadIdx.x & 31;
  // numerators (C^T r)_j: reduce-scatter over the feature lanes, lane j keeps j
  double v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = (j < DV && j < dv) ? s.c[j < DV ? j : 0] * r : 0.0;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const double keep = up ? v[i + o] : v[i];
      const double send = up ? v[i] : v[i + o];
      v[i] = keep + __shfl_xor_sync(kFull, send, o);
    }
  }
  const double nr = warp_sum(s.n * r);
  const double den = fmax(fabs(nr), exp(-s.m));
  const double h = v[0] / den;
  const double t = lane < dv ? static_cast<double>(__ldg(tail + lane)) * (h / (1.0 + exp(-h))) : 0.0;
  return static_cast<float>(warp_sum(t) + static_cast<double>(__ldg(tail + dv + 2)));
}

// Delayed readout of a token with inputs x from the state: the fp32 score.
template <int X, int DV>
__device__ __forceinline__ float state_score(const double (&x)[X], const float* __restrict__ hw, int p, int dv,
                                             const LaneState<DV>& s) {
  const float* tail = hw + static_cast<size_t>(2 * p + dv + 2) * (32 * X);
  return state_readout<DV>(hedgehog_lane(project_rows<X>(x, hw, 0, p), p), tail, dv, s);
}

// Folds a token into the state from its projections: its Hedgehog features
// (feature f in lane f), its value vector val[0, dv) and its gate
// pre-activations gi, gf (biases included).  The same arithmetic as
// state_update.
template <int DV>
__device__ __forceinline__ void state_fold(double phi, const double* val, double gi, double gf, int dv,
                                           LaneState<DV>& s) {
  const double lf = log_sigmoid(gf);
  const double m_new = fmax(lf + s.m, gi);
  const double ip = exp(gi - m_new);
  const double fp = exp(lf + s.m - m_new);
#pragma unroll
  for (int j = 0; j < DV; ++j)
    if (j < dv) s.c[j] = fp * s.c[j] + ip * (val[j] * phi);
  s.n = fp * s.n + ip * phi;
  s.m = m_new;
}

template <typename T>
__device__ __forceinline__ const T* row_ptr(const LayerArgs& a, int u, int slot) {
  return reinterpret_cast<const T*>(a.kv + (static_cast<size_t>(u) * a.NS + slot) * a.row_bytes);
}

__device__ __forceinline__ void ml_cp16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(dst)), "l"(src) : "memory");
}

// Dynamic shared memory of mlstm_step_kernel: the head's W_q, W_k, W_v rows
// (fp32), then the unit's state.
__host__ __device__ __forceinline__ int mlstm_step_smem(int p, int dv, int d) {
  return (2 * p + dv) * 2 * d * 4 + mlstm_state_doubles(p, dv) * 8;
}

// One CTA of four warps per unit.  The head's W_q, W_k, W_v rows (the
// caller's constants) are copied into shared memory before the wait for the
// previous kernel; after it, warp 2 copies the unit's state while the
// projections run.  Warps 0-2 project the step's token (write features,
// value, gates), warp 3 the boundary token's read features, all four look
// for the long-range minimum (each thread's keys loaded in one batch); then
// warp 0 folds the token into the state, reads the boundary token out and
// takes the step's decision.  The copies put every chain of dependent loads
// at one round trip.
template <typename T, int X, int DV>
__global__ void __launch_bounds__(128) mlstm_step_kernel(const LayerArgs a, const T* __restrict__ k_new,
                                                         const T* __restrict__ v_new) {
  extern __shared__ __align__(16) uint8_t ml_sm[];
  __shared__ double s_phi[32], s_val[32], s_r[32], s_g[2];
  __shared__ unsigned long long s_best[4];
  __shared__ int s_slot[4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x;
  const int h = u % a.Hkv;
  const int p = a.mp, dv = a.mdv;
  const float* hw = a.mw + static_cast<size_t>(h) * mlstm_head_floats(p, dv, a.d);
  const float* tail = hw + static_cast<size_t>(2 * p + dv + 2) * (32 * X);
  float* w_sm = reinterpret_cast<float*>(ml_sm);                                                  // [2p + dv][32 X]
  double* st_sm = reinterpret_cast<double*>(ml_sm + static_cast<size_t>(2 * p + dv) * 32 * X * 4);
  {
    const int nch = (2 * p + dv) * 32 * X / 4;   // 16-byte chunks
    for (int c = threadIdx.x; c < nch; c += 128) ml_cp16(w_sm + 4 * c, hw + 4 * c);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  // Everything below reads the previous kernels' cache, states and counters.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int N = a.layer->n_seen;
  const int ntk = a.layer->n_topk;
  if (N >= a.max_context) {   // the decode kernel that follows reports the overflow
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;
  }
  const int S = a.S, W = a.W, D = a.D, K = a.K, NS = a.NS;
  double* st = a.mstate + static_cast<size_t>(u) * mlstm_state_doubles(p, dv);
  if (warp == 2) {   // the state (16-byte multiple per unit) behind the weights
    const int nch = mlstm_state_doubles(p, dv) / 2;
    for (int c = lane; c < nch; c += 32) ml_cp16(st_sm + 2 * c, st + 2 * c);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
  } else {
    asm volatile("cp.async.wait_all;" ::: "memory");
  }
  __syncthreads();   // the weights in shared memory
  const int b = N - W - D;
  const bool has_b = b >= S;
  const int bslot = has_b ? ((D == 0) ? window_slot(b, S, W) : staging_slot(b, S, W, D)) : -1;
  const int base = topk_base(S, W, D);
  const bool scan = has_b && ntk >= K && K > 0;
  if (warp < 3) {
    double x[X];
    load_x<T, X>(k_new + static_cast<size_t>(u) * a.d, v_new + static_cast<size_t>(u) * a.d, x);
    if (warp == 0) {
      s_phi[lane] = hedgehog_lane(project_rows<X, true>(x, w_sm, p, p), p);
    } else if (warp == 1) {
      s_val[lane] = project_rows<X, true>(x, w_sm, 2 * p, dv);
    } else {
      const double g = project_rows<X>(x, hw, 2 * p + dv, 2);
      if (lane < 2) s_g[lane] = g + static_cast<double>(__ldg(tail + dv + lane));
    }
  } else if (has_b) {
    const T* row = row_ptr<T>(a, u, bslot);
    double xb[X];
    load_x<T, X>(row, row + a.d, xb);
    s_r[lane] = hedgehog_lane(project_rows<X, true>(xb, w_sm, 0, p), p);
    if ((a.flags & FLAG_DEBUG_CHECKS) && lane == 0 && a.pos[static_cast<size_t>(u) * NS + bslot] != b)
      set_error(a.err, DEVERR_STATE_MISMATCH);
  }
  if (scan) {   // minimum key (score, -position) of the long-range set as committed after step N - 1
    const int32_t* pos = a.pos + static_cast<size_t>(u) * NS + base;
    const float* score = a.score + static_cast<size_t>(u) * NS + base;
    constexpr int kB = 8;   // keys per thread per round trip
    uint64_t best = ~0ull;
    int mslot = -1;
    for (int i0 = 0; i0 < K; i0 += 128 * kB) {
      float sc[kB];
      int32_t ps[kB];
#pragma unroll
      for (int t = 0; t < kB; ++t) {
        const int i = i0 + threadIdx.x + 128 * t;
        if (i < K) { sc[t] = score[i]; ps[t] = pos[i]; }
      }
#pragma unroll
      for (int t = 0; t < kB; ++t) {
        const int i = i0 + threadIdx.x + 128 * t;
        if (i < K) {
          const uint64_t key = rank_key(sc[t], ps[t]);
          if (key < best) { best = key; mslot = base + i; }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t ok = __shfl_xor_sync(kFull, best, o);
      const int os = __shfl_xor_sync(kFull, mslot, o);
      if (ok < best) { best = ok; mslot = os; }
    }
    if (lane == 0) { s_best[warp] = best; s_slot[warp] = mslot; }
  }
  if (warp == 2) asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();   // projections, minima and the state in shared memory
  if (warp != 0) return;
  LaneState<DV> s;
  state_load<DV>(st_sm, p, dv, s);
  state_fold<DV>(s_phi[lane], s_val, s_g[0], s_g[1], dv, s);
  state_store<DV>(st, p, dv, s);
  Decision r;
  r.p = N; r.bpos = -1; r.bslot = -1; r.tgt = -1; r.evict = -1; r.sb = 0.f; r.pad[0] = r.pad[1] = 0;
  if (has_b) {
    const float sb = ranking_priority(a, u, N, state_readout<DV>(s_r[lane], tail, dv, s));
    r.bpos = b;
    r.bslot = bslot;
    r.sb = sb;
    if (ntk < K) {
      r.tgt = base + ntk;   // fill-up: next free long-range slot, nobody leaves
    } else if (K == 0) {
      r.evict = bslot;
    } else {
      uint64_t best = s_best[0];
      int mslot = s_slot[0];
#pragma unroll
      for (int w = 1; w < 4; ++w)
        if (s_best[w] < best) { best = s_best[w]; mslot = s_slot[w]; }
      if (rank_key(sb, b) > best) {
        r.tgt = mslot;
        r.evict = mslot;
      } else {
        r.evict = bslot;
      }
    }
    if ((a.flags & FLAG_DEBUG_CHECKS) && lane == 0 && sb != sb) set_error(a.err, DEVERR_NAN_SCORE);
  }
  if (lane == 0) a.dec[static_cast<size_t>(N & 1) * a.units + u] = r;
}

template <typename T, int X, int DV>
__global__ void __launch_bounds__(32 * kMlstmWarps) mlstm_prefill_kernel(const LayerArgs a, const T* __restrict__ k,
                                                                          const T* __restrict__ v, int n, int n0,
                                                                          int e0, float* __restrict__ out, int cap) {
  const int u = blockIdx.x * kMlstmWarps + (threadIdx.x >> 5);
  if (u >= a.units) return;
  const int h = u % a.Hkv;
  const int p = a.mp, dv = a.mdv, d = a.d;
  const int S = a.S, W = a.W, D = a.D;
  const float* hw = a.mw + static_cast<size_t>(h) * mlstm_head_floats(p, dv, d);
  double* st = a.mstate + static_cast<size_t>(u) * mlstm_state_doubles(p, dv);
  LaneState<DV> s;
  state_load<DV>(st, p, dv, s);
  const T* ku = k + static_cast<size_t>(u) * n * d;
  const T* vu = v + static_cast<size_t>(u) * n * d;
  // row of token t: the chunk's input, or (t < n0) its window / staging slot
  auto rows_of = [&](int t, const T*& kr, const T*& vr) {
    if (t >= n0) {
      kr = ku + static_cast<size_t>(t - n0) * d;
      vr = vu + static_cast<size_t>(t - n0) * d;
    } else {
      const int slot = (t >= n0 - W) ? window_slot(t, S, W) : staging_slot(t, S, W, D);
      kr = row_ptr<T>(a, u, slot);
      vr = kr + d;
    }
  };
  double xn[X];
  if (n > 0) load_x<T, X>(ku, vu, xn);
  for (int i = 0; i < n; ++i) {
    const int t = n0 + i;
    double x[X];
#pragma unroll
    for (int e = 0; e < X; ++e) x[e] = xn[e];
    if (i + 1 < n) load_x<T, X>(ku + static_cast<size_t>(i + 1) * d, vu + static_cast<size_t>(i + 1) * d, xn);
    const int ue = t - W - D;   // the token that becomes eligible at step t
    double xu[X];
    if (ue >= S) {
      const T *kr, *vr;
      rows_of(ue, kr, vr);
      load_x<T, X>(kr, vr, xu);
    }
    state_update<X, DV>(x, hw, p, dv, s);
    if (ue >= S) {
      const float sc = state_score<X, DV>(xu, hw, p, dv, s);
      if ((threadIdx.x & 31) == 0) out[static_cast<size_t>(u) * cap + (ue - e0)] = ranking_priority(a, u, t, sc);
    }
  }
  state_store<DV>(st, p, dv, s);
}

template <typename T, int X, int DV>
int launch_step_t(const LayerArgs& a, const void* k_new, const void* v_new, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  const int smem = mlstm_step_smem(a.mp, a.mdv, a.d);
  // The shared-memory attribute (the most any p <= 16, dv <= DV needs)
  // belongs to the current device: set once per device (devices beyond the
  // table get it on every call).
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev < 0 || dev >= kMaxDev || !attr_set[dev]) {
    if (cudaFuncSetAttribute(mlstm_step_kernel<T, X, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             mlstm_step_smem(16, DV, 16 * X)) != cudaSuccess)
      return -1;
    if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
  }
  cfg.gridDim = dim3(static_cast<unsigned>(a.units));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, mlstm_step_kernel<T, X, DV>, a, static_cast<const T*>(k_new),
                                           static_cast<const T*>(v_new));
  return e == cudaSuccess ? 0 : -1;
}

template <typename T, int X, int DV>
int launch_prefill_t(const LayerArgs& a, const void* k, const void* v, int n, int n0, int e0, float* out, int cap,
                     cudaStream_t st) {
  const int grid = (a.units + kMlstmWarps - 1) / kMlstmWarps;
  mlstm_prefill_kernel<T, X, DV><<<grid, 32 * kMlstmWarps, 0, st>>>(a, static_cast<const T*>(k),
                                                                    static_cast<const T*>(v), n, n0, e0, out, cap);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

// Shapes: d in {64, 128} (X = 4 or 8), dv <= 16 or <= 32, bf16 or fp32.
#define KVPOP_MLSTM_DISPATCH(FN, ...)                                                            \
  do {                                                                                          \
    if (dtype == 1) {                                                                           \
      if (a.d == 128) return a.mdv <= 16 ? FN<__nv_bfloat16, 8, 16>(__VA_ARGS__)                 \
                                         : FN<__nv_bfloat16, 8, 32>(__VA_ARGS__);                \
      return a.mdv <= 16 ? FN<__nv_bfloat16, 4, 16>(__VA_ARGS__) : FN<__nv_bfloat16, 4, 32>(__VA_ARGS__); \
    }                                                                                           \
    if (a.d == 128) return a.mdv <= 16 ? FN<float, 8, 16>(__VA_ARGS__) : FN<float, 8, 32>(__VA_ARGS__); \
    return a.mdv <= 16 ? FN<float, 4, 16>(__VA_ARGS__) : FN<float, 4, 32>(__VA_ARGS__);           \
  } while (0)

int launch_mlstm_step(const LayerArgs& a, int dtype, const void* k_new, const void* v_new, cudaStream_t st) {
  if (a.d != 64 && a.d != 128) return -1;
  KVPOP_MLSTM_DISPATCH(launch_step_t, a, k_new, v_new, st);
}

int launch_mlstm_prefill(const LayerArgs& a, int dtype, const void* k, const void* v, int n, int n0, int e0,
                         float* out, int cap, cudaStream_t st) {
  if (a.d != 64 && a.d != 128) return -1;
  if (n <= 0) return 0;
  KVPOP_MLSTM_DISPATCH(launch_prefill_t, a, k, v, n, n0, e0, out, cap, st);
}

#undef KVPOP_MLSTM_DISPATCH

}  // namespace kvpop
