// Parallel sparse prefill attention under the running top-k mask.
//
// KVpop page §C "Efficient Running Top-k Sparse Attention": §C.1 (one mask
// over the whole sequence: query q attends to sinks, the recent window and the
// running top-k of the eligible tokens, B = S + W + K once q is large enough)
// and §C.2 (one running cutoff per token, computed per head in O(n log n),
// evaluates the mask on the fly without an n x n mask).
//
// Cutoff.  With m = q - W - D the newest eligible position at query q, token
// j (S <= j <= n-1-W-D) is in the long-range set exactly for m in [j, c_j).
// c_j is max(j, the K-th smallest position among the tokens ranked above j),
// or "never" when fewer than K tokens rank above it: the K-th higher-ranked
// token to become eligible is the one whose arrival pushes j out, and j is
// never admitted when that happened before j itself arrived.  The page walks
// the tokens best-first with a Fenwick tree over positions; here each unit's
// eligible tokens are sorted best-first in one CTA (bitonic, shared memory),
// and one thread walks them keeping the current K-th smallest inserted
// position T: inserting a position below T moves T to its predecessor in a
// bitmap of inserted positions (T only decreases, so the walk is O(n) after
// the sort); inserting above T changes nothing.
//
// Attention.  One CTA per (unit, tile of kPaRows / G query positions) and
// its G query heads.  The CTA gathers its candidate keys once: the sinks, the
// long-range tokens still kept at its first query (c_j > m0; at most K), and
// the recent positions of its queries.  It then streams them in tiles of
// kPaKeys through shared memory with an online softmax in fp32 (FMA pipes),
// masking each (query, key) pair by the rule above.  bf16 inputs take the
// tcgen05 kernel instead (sparse_attn_tcp_kernel: persistent, one CTA per SM
// walking work items of 256 query rows, S and O accumulated in TMEM, keys
// gathered by cp.async into swizzled operand tiles); fp32 inputs keep the FMA
// kernel so that they are never rounded to a tensor-core input type.
//
// Cache build.  The tokens whose cutoff is "never" are the running top-k at
// the last prompt position; place_kept_kernel writes them to the long-range
// slots in ascending position order (what a one-chunk prefill places), so a
// whole-prompt prefill and its attention outputs share one scoring pass.
#include <cudaTypedefs.h>

#include "kvpop_prefill_attn.cuh"

namespace kvpop {

namespace {

constexpr int kCutThreads = 512;
constexpr int kPaThreads = 128;
constexpr int32_t kNever = 0x7fffffff;

__host__ __device__ inline int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// ---------------- cutoffs: sort (one CTA per unit), then walk (one warp per unit) ----------------
// The bitonic network (descending) over npow = E * kCutThreads keys in
// shared memory, with thread t holding keys t E .. t E + E - 1 in registers:
// strides below E compare within a thread, strides E .. 16 E between the
// lanes of a warp (shuffles), and only larger strides go through shared
// memory.  The same compare-exchanges as the all-shared-memory network, so
// the same order.
template <int E>
__device__ __forceinline__ void bitonic_sort_regs(uint64_t* keys, int npow) {
  const int t = threadIdx.x;
  uint64_t e[E];
#pragma unroll
  for (int k = 0; k < E; ++k) e[k] = keys[t * E + k];
  for (int kk = 2; kk <= npow; kk <<= 1) {
    int j = kk >> 1;
    if (j >= 32 * E) {   // strides across warps
#pragma unroll
      for (int k = 0; k < E; ++k) keys[t * E + k] = e[k];
      __syncthreads();
      for (; j >= 32 * E; j >>= 1) {
        for (int i = t; i < npow; i += blockDim.x) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const uint64_t x = keys[i], y = keys[ixj];
            const bool desc = (i & kk) == 0;
            if (desc ? (x < y) : (x > y)) {
              keys[i] = y;
              keys[ixj] = x;
            }
          }
        }
        __syncthreads();
      }
#pragma unroll
      for (int k = 0; k < E; ++k) e[k] = keys[t * E + k];
    }
    for (; j >= E; j >>= 1) {   // strides across the lanes of a warp: element k of thread t ^ (j / E)
      const int lm = j / E;
      const bool lower = (t & lm) == 0;
#pragma unroll
      for (int k = 0; k < E; ++k) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, e[k], lm);
        const bool desc = ((t * E + k) & kk) == 0;
        e[k] = (desc == lower) ? (e[k] > y ? e[k] : y) : (e[k] < y ? e[k] : y);
      }
    }
#pragma unroll
    for (int jj = E / 2; jj >= 1; jj >>= 1) {   // strides within the thread
      if (jj > j) continue;
#pragma unroll
      for (int k = 0; k < E; ++k) {
        if ((k & jj) != 0) continue;
        const uint64_t x = e[k], y = e[k | jj];
        const bool desc = ((t * E + k) & kk) == 0;
        if (desc ? (x < y) : (x > y)) {
          e[k] = y;
          e[k | jj] = x;
        }
      }
    }
  }
  __syncthreads();   // every thread's last shared-memory reads are done
#pragma unroll
  for (int k = 0; k < E; ++k) keys[t * E + k] = e[k];
  __syncthreads();
}

__global__ void __launch_bounds__(kCutThreads) cutoff_kernel(const float* __restrict__ scores, int score_cap,
                                                             int32_t* __restrict__ cut, int32_t* __restrict__ order,
                                                             int n, int ne, int npow, int S, uint64_t* keys_g,
                                                             int keys_global) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  int32_t* cu = cut + static_cast<size_t>(u) * n;
  uint64_t* keys = keys_global ? keys_g + static_cast<size_t>(u) * npow : reinterpret_cast<uint64_t*>(smem_raw);
  // tokens that never become eligible in the prompt
  for (int t = tid; t < n; t += blockDim.x)
    if (t < S || t >= S + ne) cu[t] = -1;
  if (ne == 0) return;
  const float* su = scores + static_cast<size_t>(u) * score_cap;
  for (int i = tid; i < npow; i += blockDim.x) keys[i] = (i < ne) ? rank_key(su[i], S + i) : 0ull;
  __syncthreads();
  // bitonic sort, descending (best first); padding keys (0) sink to the end
  if (!keys_global && npow == 16 * kCutThreads) {   // 4097 .. 8192 eligible tokens
    bitonic_sort_regs<16>(keys, npow);
  } else {
    for (int kk = 2; kk <= npow; kk <<= 1) {
      for (int j = kk >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < npow; i += blockDim.x) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const uint64_t x = keys[i], y = keys[ixj];
            const bool desc = (i & kk) == 0;
            if (desc ? (x < y) : (x > y)) {
              keys[i] = y;
              keys[ixj] = x;
            }
          }
        }
        __syncthreads();
      }
    }
  }
  // the positions in best-first order, for the walk
  int32_t* ou = order + static_cast<size_t>(u) * ne;
  for (int r = tid; r < ne; r += blockDim.x) ou[r] = static_cast<int>(0xffffffffu - static_cast<uint32_t>(keys[r]));
}

// Best-first walk of one unit per warp: T = the K-th smallest position
// among the tokens seen so far; c_j = "never" for the first K, else
// max(j, T) before j is inserted (j below T moves T to its predecessor in a
// bitmap of inserted positions).  The warp takes 32 tokens at a time (lane i
// = the i-th best of the batch; the next batch's positions load meanwhile):
// the first K set their bits and raise T together; after them the tokens at
// or above T change nothing, so one ballot finds the next one below T, the
// tokens before it take c = their own position, and only that one is
// inserted (a predecessor not in T's word is found 32 words at a time by
// ballot).  The batch's cutoffs are stored at once.
constexpr int kWalkWarps = 4;
__global__ void __launch_bounds__(32 * kWalkWarps) walk_kernel(const int32_t* __restrict__ order,
                                                               int32_t* __restrict__ cut, int n, int ne, int words,
                                                               int S, int K, int units, uint32_t* bits_g,
                                                               int bits_global, int32_t* err) {
  extern __shared__ __align__(16) uint32_t bsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * kWalkWarps + warp;
  if (u >= units || ne == 0) return;
  uint32_t* bits = bits_global ? bits_g + static_cast<size_t>(u) * words : bsm + static_cast<size_t>(warp) * words;
  for (int i = lane; i < words; i += 32) bits[i] = 0u;
  __syncwarp();
  const int32_t* ord = order + static_cast<size_t>(u) * ne;
  int32_t* cu = cut + static_cast<size_t>(u) * n;
  int T = -1;
  bool bad = false;
  int cur = lane < ne ? ord[lane] : 0;
  for (int r0 = 0; r0 < ne && !bad; r0 += 32) {
    const int nxt = r0 + 32 + lane < ne ? ord[r0 + 32 + lane] : 0;   // the next batch, in flight meanwhile
    const int lim = min(32, ne - r0);
    const bool valid = lane < lim;
    int myc = cur;   // K = 0: c = j
    if (K > 0) {
      // the batch's tokens among the first K: "never", their bits set, T = max
      const bool first_k = valid && r0 + lane < K;
      if (__any_sync(0xffffffffu, first_k)) {
        if (first_k) {
          const int idx = cur - S;
          atomicOr(&bits[idx >> 5], 1u << (idx & 31));
          myc = kNever;
        }
        int tm = first_k ? cur : -1;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tm = max(tm, __shfl_xor_sync(0xffffffffu, tm, o));
        T = max(T, tm);
        __syncwarp();
      }
      // the rest in best-first order: up to the next token below T, c = max(j, T) = j
      int x = r0 >= K ? 0 : K - r0;
      while (x < lim) {
        const uint32_t below = __ballot_sync(0xffffffffu, valid && lane >= x && cur < T);
        const int xi = below != 0u ? __ffs(below) - 1 : lim;
        if (lane >= x && lane < xi) myc = max(cur, T);
        if (xi == lim) break;
        // token xi is below T: c = T, insert it, T moves to its predecessor
        const int pos = __shfl_sync(0xffffffffu, cur, xi);
        if (lane == xi) myc = T;
        const int idx = pos - S;
        if (lane == 0) bits[idx >> 5] |= 1u << (idx & 31);
        __syncwarp();
        const int ti = T - S;
        const int w = ti >> 5;
        const uint32_t m = bits[w] & ((1u << (ti & 31)) - 1u);
        if (m != 0u) {
          T = S + (w << 5) + 31 - __clz(m);
        } else {
          bool found = false;
          for (int base = w - 1; base >= 0 && !found; base -= 32) {
            const int wi = base - lane;
            const uint32_t bv = wi >= 0 ? bits[wi] : 0u;
            const uint32_t bal = __ballot_sync(0xffffffffu, bv != 0u);
            if (bal != 0u) {
              const int l = __ffs(bal) - 1;   // the lowest lane holds the highest word
              T = S + ((base - l) << 5) + 31 - __clz(__shfl_sync(0xffffffffu, bv, l));
              found = true;
            }
          }
          if (!found) {   // cannot happen: pos < T was just inserted
            bad = true;
            break;
          }
        }
        x = xi + 1;
      }
    }
    if (!bad && valid) cu[cur] = myc;
    cur = nxt;
  }
  if (bad && lane == 0) set_error(err, DEVERR_STATE_MISMATCH);
}

// ---------------- attention: one CTA per (query tile, unit) ----------------
struct PaArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  const int32_t* cut;
  int n, S, W, D, G, Hq, Hkv, qt, cand_cap;
  float scale_log2;   // log2(e) / sqrt(d): logits in base-2 units
  int32_t* err;       // device error word (bounded waits that give up)
};

template <typename T> struct PaIo;
template <> struct PaIo<float> {
  static __device__ __forceinline__ void load8(const float* p, float* o) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
  static __device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
};

// Candidate keys of a tile of query positions [q0, q1) with m0 = q0 - W - D,
// in ascending position: the sinks, the long-range tokens still kept at m0
// (c_j > m0; at most K of them) and the recent block [max(S, m0 + 1), q1).
// Every key a query of the tile may attend to is among them.  Block-wide
// (all NT threads); returns the count (at most cap).  Each thread scans 8
// consecutive positions per round (8 cutoff loads in flight), and one block
// scan per NT * 8 positions places the kept ones.
template <int NT>
__device__ int gather_candidates(int* cand, int* wtot, const int32_t* cu, int S, int m0, int q1, int cap) {
  constexpr int R = 8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ns = min(S, q1);
  for (int i = tid; i < ns; i += NT) cand[i] = i;
  int count = ns;
  for (int base = S; base <= m0; base += NT * R) {
    const int j0 = base + tid * R;
    int c[R];
#pragma unroll
    for (int r = 0; r < R; ++r) c[r] = (j0 + r <= m0) ? cu[j0 + r] : 0;
    unsigned mine = 0u;
#pragma unroll
    for (int r = 0; r < R; ++r) mine |= (j0 + r <= m0 && c[r] > m0) ? (1u << r) : 0u;
    const int cnt = __popc(mine);
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane == 31) wtot[warp] = inc;
    __syncthreads();
    int off = count, total = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
      const int t = wtot[w];
      off += (w < warp) ? t : 0;
      total += t;
    }
    off += inc - cnt;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if ((mine >> r) & 1u) {
        if (off < cap) cand[off] = j0 + r;
        ++off;
      }
    }
    count += total;
    __syncthreads();
  }
  const int r0 = max(S, m0 + 1);
  const int nr = max(0, q1 - r0);
  for (int i = tid; i < nr; i += NT)
    if (count + i < cap) cand[count + i] = r0 + i;
  count += nr;
  __syncthreads();
  return min(count, cap);   // count <= cap always: S + K + qt + W + D bounds it
}

template <int DH>
struct PaSmem {
  static constexpr int KS = DH + 4;                 // padded key/value row (floats)
  static constexpr int PS = kPaKeys + 1;            // padded probability row (floats)
  static constexpr size_t Q_OFF = 0;
  static constexpr size_t K_OFF = Q_OFF + sizeof(float) * kPaRows * DH;
  static constexpr size_t V_OFF = K_OFF + sizeof(float) * kPaKeys * KS;
  static constexpr size_t P_OFF = V_OFF + sizeof(float) * kPaKeys * KS;
  static constexpr size_t POS_OFF = P_OFF + sizeof(float) * kPaRows * PS;
  static constexpr size_t CUT_OFF = POS_OFF + sizeof(int) * kPaKeys;
  static constexpr size_t WT_OFF = CUT_OFF + sizeof(int) * kPaKeys;
  static constexpr size_t CAND_OFF = WT_OFF + 16 * sizeof(int);
  static size_t bytes(int cand_cap) { return CAND_OFF + sizeof(int) * static_cast<size_t>(cand_cap); }
};

template <typename T, int DH>
__global__ void __launch_bounds__(kPaThreads) sparse_attn_kernel(PaArgs p) {
  using SM = PaSmem<DH>;
  constexpr int NC = DH / 32;   // float4 chunks of a row per thread in P.V
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* Qs = reinterpret_cast<float*>(smem_raw + SM::Q_OFF);
  float* Ks = reinterpret_cast<float*>(smem_raw + SM::K_OFF);
  float* Vs = reinterpret_cast<float*>(smem_raw + SM::V_OFF);
  float* Ps = reinterpret_cast<float*>(smem_raw + SM::P_OFF);
  int* kpos = reinterpret_cast<int*>(smem_raw + SM::POS_OFF);
  int* kcut = reinterpret_cast<int*>(smem_raw + SM::CUT_OFF);
  int* wtot = reinterpret_cast<int*>(smem_raw + SM::WT_OFF);
  int* cand = reinterpret_cast<int*>(smem_raw + SM::CAND_OFF);

  const int tid = threadIdx.x;
  const int rg = tid >> 3, kg = tid & 7;
  const int u = blockIdx.y;
  const int b = u / p.Hkv, hk = u % p.Hkv;
  const int n = p.n, S = p.S, WD = p.W + p.D, G = p.G;
  const int q0 = blockIdx.x * p.qt;
  const int q1 = min(n, q0 + p.qt);
  const T* qg = static_cast<const T*>(p.q);
  const T* kgp = static_cast<const T*>(p.k) + static_cast<size_t>(u) * n * DH;
  const T* vgp = static_cast<const T*>(p.v) + static_cast<size_t>(u) * n * DH;
  const int32_t* cu = p.cut + static_cast<size_t>(u) * n;

  // queries of the tile, pre-scaled to base-2 logits
  for (int c = tid; c < kPaRows * (DH / 8); c += kPaThreads) {
    const int row = c / (DH / 8), ch = c % (DH / 8);
    const int qpos = q0 + row / G, g = row % G;
    float x[8];
    if (qpos < q1) {
      PaIo<T>::load8(qg + ((static_cast<size_t>(b) * p.Hq + hk * G + g) * n + qpos) * DH + ch * 8, x);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    float4* dst = reinterpret_cast<float4*>(Qs + row * DH + ch * 8);
    dst[0] = make_float4(x[0] * p.scale_log2, x[1] * p.scale_log2, x[2] * p.scale_log2, x[3] * p.scale_log2);
    dst[1] = make_float4(x[4] * p.scale_log2, x[5] * p.scale_log2, x[6] * p.scale_log2, x[7] * p.scale_log2);
  }

  const int count = gather_candidates<kPaThreads>(cand, wtot, cu, S, q0 - WD, q1, p.cand_cap);

  float4 o[4][NC];
  float mrow[4], lrow[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    mrow[r] = -INFINITY;
    lrow[r] = 0.f;
#pragma unroll
    for (int i = 0; i < NC; ++i) o[r][i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  int rq[4], rm[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    rq[r] = q0 + (4 * rg + r) / G;
    rm[r] = rq[r] - WD;
  }

  for (int t0 = 0; t0 < count; t0 += kPaKeys) {
    if (tid < kPaKeys) {
      const int idx = t0 + tid;
      const int j = idx < count ? cand[idx] : -1;
      kpos[tid] = j;
      kcut[tid] = j >= 0 ? cu[j] : 0;
    }
    for (int c = tid; c < kPaKeys * (DH / 8); c += kPaThreads) {
      const int key = c / (DH / 8), ch = c % (DH / 8);
      const int idx = t0 + key;
      float xk[8], xv[8];
      if (idx < count) {
        const int j = cand[idx];
        PaIo<T>::load8(kgp + static_cast<size_t>(j) * DH + ch * 8, xk);
        PaIo<T>::load8(vgp + static_cast<size_t>(j) * DH + ch * 8, xv);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xk[e] = xv[e] = 0.f;
      }
      float4* dk = reinterpret_cast<float4*>(Ks + key * SM::KS + ch * 8);
      float4* dv = reinterpret_cast<float4*>(Vs + key * SM::KS + ch * 8);
      dk[0] = make_float4(xk[0], xk[1], xk[2], xk[3]);
      dk[1] = make_float4(xk[4], xk[5], xk[6], xk[7]);
      dv[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
      dv[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
    }
    __syncthreads();

    // logits of the thread's 4 rows x 4 keys (keys kg, kg+8, kg+16, kg+24)
    float s[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i) s[r][i] = 0.f;
#pragma unroll 4
    for (int dd = 0; dd < DH; dd += 4) {
      float4 qv[4], kv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) qv[r] = *reinterpret_cast<const float4*>(Qs + (4 * rg + r) * DH + dd);
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = *reinterpret_cast<const float4*>(Ks + (kg + 8 * i) * SM::KS + dd);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          s[r][i] = fmaf(qv[r].x, kv[i].x, s[r][i]);
          s[r][i] = fmaf(qv[r].y, kv[i].y, s[r][i]);
          s[r][i] = fmaf(qv[r].z, kv[i].z, s[r][i]);
          s[r][i] = fmaf(qv[r].w, kv[i].w, s[r][i]);
        }
    }

    // mask (running top-k rule) and online softmax
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float tmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int key = kg + 8 * i;
        const int j = kpos[key];
        const bool vis = j >= 0 && rq[r] < q1 && j <= rq[r] && (j < S || j > rm[r] || kcut[key] > rm[r]);
        s[r][i] = vis ? s[r][i] : -INFINITY;
        tmax = fmaxf(tmax, s[r][i]);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
      const float mnew = fmaxf(mrow[r], tmax);
      const float alpha = (mnew == -INFINITY) ? 1.f : exp2f(mrow[r] - mnew);
      float psum = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float pv = (s[r][i] == -INFINITY) ? 0.f : exp2f(s[r][i] - mnew);
        psum += pv;
        Ps[(4 * rg + r) * SM::PS + kg + 8 * i] = pv;
      }
      psum += __shfl_xor_sync(0xffffffffu, psum, 1);
      psum += __shfl_xor_sync(0xffffffffu, psum, 2);
      psum += __shfl_xor_sync(0xffffffffu, psum, 4);
      lrow[r] = lrow[r] * alpha + psum;
      mrow[r] = mnew;
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        o[r][i].x *= alpha;
        o[r][i].y *= alpha;
        o[r][i].z *= alpha;
        o[r][i].w *= alpha;
      }
    }
    __syncthreads();

    // O += P . V  (the thread's rows x its column chunks kg, kg+8, ...)
#pragma unroll 4
    for (int key = 0; key < kPaKeys; ++key) {
      float pr[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) pr[r] = Ps[(4 * rg + r) * SM::PS + key];
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const float4 vv = *reinterpret_cast<const float4*>(Vs + key * SM::KS + (kg + 8 * i) * 4);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          o[r][i].x = fmaf(pr[r], vv.x, o[r][i].x);
          o[r][i].y = fmaf(pr[r], vv.y, o[r][i].y);
          o[r][i].z = fmaf(pr[r], vv.z, o[r][i].z);
          o[r][i].w = fmaf(pr[r], vv.w, o[r][i].w);
        }
      }
    }
    __syncthreads();
  }

  T* og = static_cast<T*>(p.out);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = 4 * rg + r;
    const int qpos = rq[r], g = row % G;
    if (qpos >= q1) continue;
    const size_t rowi = (static_cast<size_t>(b) * p.Hq + hk * G + g) * n + qpos;
    const float inv = 1.f / lrow[r];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      const float4 v4 = make_float4(o[r][i].x * inv, o[r][i].y * inv, o[r][i].z * inv, o[r][i].w * inv);
      PaIo<T>::store4(og + rowi * DH + (kg + 8 * i) * 4, v4);
    }
    if (p.lse != nullptr && kg == 0) p.lse[rowi] = (mrow[r] + log2f(lrow[r])) * 0.69314718055994531f;
  }
}

// ---------------- tcgen05 and copy helpers ----------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Shared-memory matrix descriptor, no swizzle (start, leading and stride
// byte offsets in 16-byte units; descriptor version 1).
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, M x N,
// B K-major (b_mn = 0) or MN-major (b_mn = 1), A K-major.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tc_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
         "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])),
         "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
         "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
         "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
         "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
         "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
         "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
         "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
         "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// 2^x with the hardware's approximate base-2 exponential (ftz; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Shared-memory matrix descriptor, 128-byte swizzle (atoms of 8 rows x 128
// bytes, 1024-byte aligned; start, leading and stride byte offsets in 16-byte
// units; descriptor version 1, layout type 2).  K-major: stride offset =
// 8-row group stride, leading offset unused (1), and the start moves by 32
// bytes per 16 elements of K inside the atom.  MN-major: leading offset =
// stride between 64-element groups of MN, stride offset = 8-row group stride
// along K.
__device__ __forceinline__ uint64_t tc_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return tc_desc(saddr, lbo, sbo) | (2ull << 61);
}
// D (+)= A B with A and B in shared memory (descriptors).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
// D (+)= A B with A in TMEM (row m = lane m, K pairs of bf16 per 32-bit
// column) and B in shared memory (descriptor).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n"
      :: "r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
// 16 consecutive 32-bit columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tc_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};"
      :: "r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
         "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// ---------------- bf16 attention on tcgen05: persistent, two row blocks per work item ----------------
// One CTA per SM walks its share of the work items (unit, 256 query rows =
// 256 / G positions x G heads), items blockIdx.x, blockIdx.x + gridDim.x, ...
// in order.  Warp-specialized and pipelined through mbarriers, with the
// pipeline running on across item boundaries (a global tile counter T picks
// every stage, buffer and parity):
//   copy warps 8-11 gather the next item's candidate keys while the current
//     item's last tiles are still being computed, then each 64-key tile's K
//     and V rows by cp.async into the 128-byte-swizzled operand layout (NST
//     stages; each thread's copies arrive on the stage's mbarrier as they
//     land); mask warps 12-13 build each tile's mask (64 key bits per query
//     position);
//   one thread of warp 14 (block 0) and one of warp 15 (block 1) issue each
//     block's MMAs: S(T), S(T + 1), then per tile O += P V(T) and S(T + 2);
//     each tile's K and V serve both blocks.  The same thread loads its
//     block's Q rows of the next item by TMA as soon as the current item's
//     last S has read them;
//   softmax warps 0-3 (block 0) and 4-7 (block 1): thread = query row = TMEM
//     lane; each item ends with its rows' epilogue, while the next item's
//     first S tiles are already computed.
// Q (A of S = Q K^T) sits in shared memory; S is double-buffered in TMEM per
// block; the softmax writes P(T) in bf16 over S(T) (A of P V from TMEM).  One
// thread's MMAs run in issue order, so S(T + 2) overwrites that buffer only
// after P V(T) has read it.  An O rescale (rare: lazy threshold) waits for
// the P V before.  TMEM columns: O[block] at block * DH, S[block][buf] at
// 2 DH + 64 (2 block + buf).  Block X holds query positions X * 128 / G ..
// (X + 1) * 128 / G - 1 of the item; its row r is head r / (128 / G) at
// position r % (128 / G), so each head's rows are one TMA box of Q.  Every
// mbarrier that a role may wait on twice in a row without an intervening
// handoff is per buffer, so parity waits never alias.

// 64 consecutive fp32 columns of this thread's TMEM lane in one load, waited
// for inside the same statement (warp-collective).
__device__ __forceinline__ void tc_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {"
      "%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, "
      "%18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, "
      "%34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, "
      "%50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63"
      "}, [%64];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

constexpr int kT2Rows = 256;
// Lazy rescale threshold (log2 units): the running max of a row moves only
// when a tile's max exceeds it by 2^20.  A rescale of O waits for the P V in
// flight, so it must be rare; weights then stay below 2^20, far inside the
// range of the fp32 accumulators (and of bf16 P, whose precision is
// relative).
constexpr float kT2Lazy = 20.0f;
constexpr int kT2Keys = 64;
constexpr int kT2Threads = 16 * 32;
constexpr int kT2Prod = 8;          // first of the 4 copy warps
constexpr int kT2Mask = 12;         // first of the 2 mask warps
constexpr int kT2Mma = 14;          // MMA warps: one per row block
constexpr uint32_t kT2Cols = 512;
constexpr int kT2Ring = 8;          // tile counts of items in flight (more than NST + 1 items)
constexpr int kT2CopyBar = 1;       // named barrier of the 128 copy threads

// Shared memory: Q of both blocks, then NST stages each holding the tile's K
// then V, all in the K-major / MN-major 128-byte-swizzled layout: rows of 64
// columns (128 bytes) in swizzle atoms of 8 rows x 128 bytes.  Q: per block
// DH / 64 groups of 16 atoms (128 rows); K and V: DH / 64 groups of 8 atoms
// (64 keys).  Then the masks, the barriers, a few words, and the candidate
// positions of two items (the current one and the next, gathered ahead).
template <int DH, int NST>
struct T2Smem {
  static constexpr int NGRP = DH / 64;                                           // 64-column groups per row
  static constexpr size_t QGRP = 128 * 128;                                      // one group of one Q block: 16 KB
  static constexpr size_t QBLK = NGRP * QGRP;
  static constexpr size_t Q_OFF = 0;
  static constexpr size_t GRP = static_cast<size_t>(kT2Keys) * 128;              // one group of one tile: 8 KB
  static constexpr size_t KV_TILE = NGRP * GRP;
  static constexpr size_t STAGE = 2 * KV_TILE;
  static constexpr size_t KV_OFF = Q_OFF + 2 * QBLK;                            // [stage][K, V]
  static constexpr size_t META_OFF = KV_OFF + NST * STAGE;                      // [stage][query position] key masks
  static constexpr int META_INTS = 2 * kT2Rows + 4;                              // 2 words per position (256 / G at most), then the full-tile flag
  static constexpr size_t BAR_OFF = META_OFF + sizeof(int) * NST * META_INTS;
  static constexpr int NBAR = 3 * NST + 4 + 4 + 2 + 2 + 2 + kT2Ring + 2;
  static constexpr size_t MISC_OFF = BAR_OFF + 8 * NBAR;                        // TMEM address, abort flag, tile-count ring, warp totals
  static constexpr size_t EXC_OFF = MISC_OFF + 128;                             // gather scratch: the item's evicted long-range keys
  static constexpr size_t CAND_OFF = EXC_OFF + sizeof(int) * kT2Rows;           // [item % 2][cand_cap] positions
  static_assert(BAR_OFF % 8 == 0 && STAGE % 1024 == 0 && KV_OFF % 1024 == 0 && META_OFF % 16 == 0 &&
                    2 + kT2Ring + 8 <= 32,
                "shared-memory layout");
  // at least 116 KB: one CTA per SM, which then holds all 512 TMEM columns
  static size_t bytes(int cand_cap) {
    const size_t bb = CAND_OFF + 2 * sizeof(int) * static_cast<size_t>(cand_cap);
    return bb > 116 * 1024 ? bb : 116 * 1024;
  }
};

// 32 x 32 bit-matrix transpose across a warp: lane i holds row i (bit j =
// column j) on entry and column i (bit j = row j) on return.  Five rounds
// swap off-diagonal blocks of 16, 8, 4, 2 and 1 between lanes i and i ^ k.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
  constexpr uint32_t kMask[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int k = 16 >> s;
    const uint32_t m = kMask[s];
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, k);
    x = (lane & k) ? ((x & ~m) | ((y >> k) & m)) : ((x & m) | ((y << k) & ~m));
  }
  return x;
}
// Bits a..b (inclusive) of a 32-bit word, clipped to 0..31; 0 when empty.
__device__ __forceinline__ uint32_t bit_range32(int a, int b) {
  if (a > b || a > 31 || b < 0) return 0u;
  return (0xffffffffu >> (31 - min(b, 31))) & (0xffffffffu << max(a, 0));
}
// Named barrier over `nthreads` threads (whole warps); the second form
// returns whether any participating thread passed true.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r) : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads) : "memory");
  return r != 0;
}
// 32 bytes to global memory in one store (the address 32-byte aligned).
__device__ __forceinline__ void st_global_v8(void* ptr, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               :: "l"(ptr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
// Non-blocking test of an mbarrier phase (acquire on success).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Test of an mbarrier phase that may suspend the thread (no issue slots) for
// up to about `ns` nanoseconds while the phase is incomplete.
__device__ __forceinline__ bool mbar_try_wait_ns(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(ns) : "memory");
  return ok != 0;
}
// One box of a 3-D tensor map into shared memory (no multicast), completion
// counted in bytes on the mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

// The candidates of one work item (the keys gather_candidates lists),
// computed by the 128 copy threads (ptid 0..127) alone, synchronised by
// named barrier kT2CopyBar, in the order: sinks, the long-range keys still
// kept at the item's last query (visible to all its positions), the ones
// evicted inside the item's range (at most one per position, kept in `exc`
// until the scan ends), then the recent block; so that only the last few
// tiles of an item need a mask.  Each warp scans 32 x R consecutive cutoffs
// per round with coalesced loads (lane i reads position base + 32 r + i),
// ballots the kept ones and places them after the earlier warps' (one scan
// over the four warps' two totals per round of 128 x R positions).  Entry:
// the position j, or, with `packed` (prompts of at most 65,535 tokens),
// j | min(max(j, c_j), 65535) << 16, so that the mask needs no cutoff load
// (positions and query indices stay below 65,535, so the clamp never changes
// q - W - D < max(j, c_j)).  Returns the count (at most cap).
__device__ __forceinline__ uint32_t cand_entry(int j, int c, bool packed) {
  return packed ? static_cast<uint32_t>(j) | (static_cast<uint32_t>(min(max(j, c), 65535)) << 16)
                : static_cast<uint32_t>(j);
}
__device__ __forceinline__ int gather_candidates_copy(uint32_t* cand, uint32_t* exc, int* wtot, const int32_t* cu,
                                                      int S, int m0, int m1, int q1, int cap, int ptid, bool packed) {
  constexpr int NT = 128, R = 8;
  const int lane = ptid & 31, w = ptid >> 5;
  const int ns = min(S, q1);
  for (int i = ptid; i < ns; i += NT) cand[i] = cand_entry(i, 0, packed);
  int na = ns, ne = 0;   // entries placed: sinks and kept keys / evicted keys
  const uint32_t lt = (1u << lane) - 1u;
  for (int base = S; base <= m0; base += NT * R) {
    const int wb = base + w * 32 * R;
    int c[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = wb + 32 * r + lane;
      c[r] = j <= m0 ? cu[j] : 0;
    }
    uint32_t ba[R], be[R];
    int ta = 0, te = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = wb + 32 * r + lane;
      ba[r] = __ballot_sync(0xffffffffu, j <= m0 && c[r] > m1);
      be[r] = __ballot_sync(0xffffffffu, j <= m0 && c[r] > m0 && c[r] <= m1);
      ta += __popc(ba[r]);
      te += __popc(be[r]);
    }
    if (lane == 0) {
      wtot[w] = ta;
      wtot[4 + w] = te;
    }
    named_bar_sync(kT2CopyBar, NT);
    int oa = na, oe = ne, sa = 0, se = 0;
#pragma unroll
    for (int x = 0; x < NT / 32; ++x) {
      const int xa = wtot[x], xe = wtot[4 + x];
      oa += (x < w) ? xa : 0;
      oe += (x < w) ? xe : 0;
      sa += xa;
      se += xe;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = wb + 32 * r + lane;
      if ((ba[r] >> lane) & 1u) {
        const int o = oa + __popc(ba[r] & lt);
        if (o < cap) cand[o] = cand_entry(j, c[r], packed);
      }
      if ((be[r] >> lane) & 1u) {
        const int o = oe + __popc(be[r] & lt);
        if (o < kT2Rows) exc[o] = cand_entry(j, c[r], packed);
      }
      oa += __popc(ba[r]);
      oe += __popc(be[r]);
    }
    na += sa;
    ne += se;
    named_bar_sync(kT2CopyBar, NT);   // wtot is rewritten next round; exc complete
  }
  ne = min(ne, kT2Rows);   // at most m1 - m0 < qt <= kT2Rows evictions
  for (int i = ptid; i < ne; i += NT)
    if (na + i < cap) cand[na + i] = exc[i];
  int count = na + ne;
  const int r0 = max(S, m0 + 1);
  const int nr = max(0, q1 - r0);
  for (int i = ptid; i < nr; i += NT)
    if (count + i < cap) cand[count + i] = cand_entry(r0 + i, packed ? cu[r0 + i] : 0, packed);
  count += nr;
  named_bar_sync(kT2CopyBar, NT);
  return min(count, cap);   // count <= cap always: S + K + qt + W + D bounds it
}

// A work item: 256 / G query positions [q0, q1) of unit u (batch row b, KV head hk).
struct T2Item {
  int u, b, hk, q0, q1;
};
__device__ __forceinline__ T2Item t2_item(const PaArgs& p, int ntq, int it) {
  T2Item w;
  w.u = it / ntq;
  w.b = w.u / p.Hkv;
  w.hk = w.u % p.Hkv;
  w.q0 = (it % ntq) * p.qt;
  w.q1 = min(p.n, w.q0 + p.qt);
  return w;
}

template <int DH, int NST>
__global__ void __launch_bounds__(kT2Threads, 1)
sparse_attn_tcp_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ PaArgs p, int nitems) {
  using SM = T2Smem<DH, NST>;
  constexpr uint32_t kIdescS = tc_idesc(128, kT2Keys, 0);
  constexpr uint32_t kIdescPV = tc_idesc(128, DH, 1);
  extern __shared__ __align__(1024) uint8_t smem_t2[];
  const uint32_t sbase = smem_u32(smem_t2);
  if ((sbase & 1023u) != 0u) {   // the swizzle atoms need 1024-byte alignment
    if (threadIdx.x == 0) set_error(p.err, DEVERR_BAD_INDEX);
    return;
  }
  int* meta = reinterpret_cast<int*>(smem_t2 + SM::META_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_t2 + SM::BAR_OFF);
  uint64_t* kv_full = bars;                       // [stage], 128 copy-thread arrivals as their copies land
  uint64_t* kv_free = bars + NST;                 // [stage], one MMA commit per row block
  uint64_t* meta_full = bars + 2 * NST;           // [stage], the 2 mask warps
  uint64_t* s_full = bars + 3 * NST;              // [block][buf], MMA commit of S(T)
  uint64_t* p_full = s_full + 4;                  // [block][buf], 128 softmax arrivals: P(T) over S(T)
  uint64_t* o_done = p_full + 4;                  // [block], MMA commit after each P V
  uint64_t* q_full = o_done + 2;                  // [block], the block's Q rows of an item landed (TMA bytes)
  uint64_t* q_free = q_full + 2;                  // [block], MMA commit after an item's last S
  uint64_t* item_full = q_free + 2;               // [item % ring], the item's candidates and tile count are ready
  uint64_t* cand_free = item_full + kT2Ring;      // [item % 2], the mask warps are done with the item's candidates
  int* misc = reinterpret_cast<int*>(smem_t2 + SM::MISC_OFF);
  uint32_t* taddr_s = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = misc + 1;
  int* count_ring = misc + 2;                     // [item % ring] candidate count of the item
  int* wtot = misc + 2 + kT2Ring;                 // copy warps' two totals each (gather scan)
  uint32_t* exc = reinterpret_cast<uint32_t*>(smem_t2 + SM::EXC_OFF);

  uint32_t* cand2 = reinterpret_cast<uint32_t*>(smem_t2 + SM::CAND_OFF);   // item i's candidates at cand2 + (i & 1) * cand_cap

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.n, S = p.S, WD = p.W + p.D, G = p.G;
  const int ntq = (n + p.qt - 1) / p.qt;
  const int PB = 128 / G;                          // query positions per row block
  const bool packed = n <= 65535;                  // candidate entries carry max(j, c_j) (cand_entry)
  const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.k);
  const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(p.v);

  if (warp == kT2Mma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(taddr_s)), "r"(kT2Cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 128);
      mbar_init(&kv_free[i], 2);
      mbar_init(&meta_full[i], kT2Mma - kT2Mask);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&o_done[i], 1);
      mbar_init(&q_full[i], 1);
      mbar_init(&q_free[i], 1);
    }
    for (int i = 0; i < kT2Ring; ++i) mbar_init(&item_full[i], 1);
    for (int i = 0; i < 2; ++i) mbar_init(&cand_free[i], kT2Mma - kT2Mask);
    *abort_flag = 0;
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *taddr_s;
  constexpr uint32_t kColS = 2 * DH;   // TMEM: O[block] at block * DH, S[block][buf] at kColS + 64 (2 block + buf)

  // bounded wait; on expiry every role stops at its next check
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    if (lane == 0) set_error(p.err, DEVERR_TIMEOUT);
    *abort_flag = 1;
    return false;
  };
  auto ntiles_of = [](int count) { return (count + kT2Keys - 1) / kT2Keys; };

  if (warp >= kT2Prod && warp < kT2Mask) {
    // ---------------- copy warps: candidates, then K and V tiles ----------------
    // Their loop is bound by the load/store unit's rate for cp.async; the
    // masks are built by other warps, so no shared-memory access of theirs
    // queues behind these copies.  The candidates of item i + 1 are gathered
    // once item i's first NST tiles are issued (or after all of them, if it
    // has fewer), into the buffer of item i - 1 (released by the mask
    // warps); the softmax and MMA roles only need the count, kept in a ring.
    // Every named barrier and every exit is taken by all 128 threads alike: a
    // thread whose wait failed skips its work but keeps the same path.
    const int ptid = (warp - kT2Prod) * 32 + lane;
    bool failed = false;
    auto gather = [&](int i) {   // item i's candidates into its buffer; count to the ring
      const T2Item w = t2_item(p, ntq, blockIdx.x + i * gridDim.x);
      const int count = gather_candidates_copy(cand2 + (i & 1) * p.cand_cap, exc, wtot,
                                               p.cut + static_cast<size_t>(w.u) * n, S, w.q0 - WD, w.q1 - 1 - WD,
                                               w.q1, p.cand_cap, ptid, packed);
      if (ptid == 0) {
        count_ring[i % kT2Ring] = count;
        mbar_arrive(&item_full[i % kT2Ring]);
      }
      return count;
    };
    int next_count = gather(0);
    int T = 0;
    for (int i = 0;; ++i) {
      const int it = blockIdx.x + i * gridDim.x;
      if (it >= nitems) break;
      const T2Item w = t2_item(p, ntq, it);
      const bool has_next = it + static_cast<int>(gridDim.x) < nitems;
      const uint32_t* cand = cand2 + (i & 1) * p.cand_cap;
      const int count = next_count;
      const int nt = ntiles_of(count);
      const int gat = min(NST, nt);
      const __nv_bfloat16* kgp = kbase + static_cast<size_t>(w.u) * n * DH;
      const __nv_bfloat16* vgp = vbase + static_cast<size_t>(w.u) * n * DH;
      for (int t = 0; t <= nt; ++t) {
        if (t == gat && has_next) {
          const bool good = failed || i == 0 || wait(&cand_free[(i - 1) & 1], ((i - 1) >> 1) & 1);
          if (named_bar_or(kT2CopyBar, 128, failed || !good || *abort_flag != 0))
            failed = true;
          else
            next_count = gather(i + 1);
        }
        if (t == nt) break;
        const int st = T % NST;
        ++T;
        if (failed || (T > NST && !wait(&kv_free[st], (((T - 1) / NST) - 1) & 1))) {
          failed = true;
          continue;
        }
        // The tile's K and V rows by cp.async into the swizzled layout: lane
        // = 16-byte chunk of a 256-byte row (two rows per warp instruction),
        // chunk c of key r at group c / 8, atom r / 8, row r % 8, position
        // (c % 8) ^ (r % 8).  Past the candidates: zero-filled.  Each thread
        // then arrives on kv_full[stage] when its copies have landed.
        constexpr int CPR = DH / 8;                       // 16-byte chunks per row
        const uint32_t kb = sbase + static_cast<uint32_t>(SM::KV_OFF + st * SM::STAGE);
#pragma unroll
        for (int x = ptid; x < kT2Keys * CPR; x += 128) {
          const int key = x / CPR, c = x % CPR;
          const int kidx = t * kT2Keys + key;
          const int jj = kidx < count ? static_cast<int>(packed ? cand[kidx] & 0xffffu : cand[kidx]) : -1;
          const size_t off = jj >= 0 ? static_cast<size_t>(jj) * DH + c * 8 : 0;
          const uint32_t so = static_cast<uint32_t>((c >> 3) * SM::GRP + (key >> 3) * 1024 + (key & 7) * 128 +
                                                    (((c & 7) ^ (key & 7)) << 4));
          cp_async16(kb + so, kgp + off, jj >= 0 ? 16 : 0);
          cp_async16(kb + static_cast<uint32_t>(SM::KV_TILE) + so, vgp + off, jj >= 0 ? 16 : 0);
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" :: "r"(smem_u32(&kv_full[st])) : "memory");
      }
      if (named_bar_or(kT2CopyBar, 128, failed || *abort_flag != 0)) break;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // nothing lands after the CTA's last barrier
  } else if (warp >= kT2Mask && warp < kT2Mma) {
    // ---------------- mask warps ----------------
    const int mw = warp - kT2Mask;
    int T = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int it = blockIdx.x + i * gridDim.x;
      if (it >= nitems) break;
      if (!__all_sync(0xffffffffu, wait(&item_full[i % kT2Ring], (i / kT2Ring) & 1))) break;
      const T2Item w = t2_item(p, ntq, it);
      const int q0 = w.q0, q1 = w.q1;
      const int count = count_ring[i % kT2Ring];
      const int nt = ntiles_of(count);
      const uint32_t* cand = cand2 + (i & 1) * p.cand_cap;
      const int32_t* cu = p.cut + static_cast<size_t>(w.u) * n;
      // lane's keys 32 h + lane of tile t: position (-1 past the candidates) and max(position, cutoff)
      auto load_keys = [&](int t, int (&jj)[2], int (&mm)[2]) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int idx = t * kT2Keys + 32 * h + lane;
          const uint32_t e = idx < count ? cand[idx] : 0xffffffffu;
          jj[h] = idx < count ? static_cast<int>(packed ? e & 0xffffu : e) : -1;
          mm[h] = jj[h] < 0 ? 0 : packed ? static_cast<int>(e >> 16) : max(jj[h], cu[jj[h]]);
        }
      };
      int jn[2], mn[2];   // the next tile's keys, loaded one tile ahead (long prompts read the cutoffs from global memory)
      load_keys(0, jn, mn);
      for (int t = 0; t < nt; ++t, ++T) {
        const int st = T % NST;
        if (!__all_sync(0xffffffffu, T < NST || wait(&kv_free[st], ((T / NST) - 1) & 1))) {
          ok = false;
          break;
        }
        const int jh[2] = {jn[0], jn[1]}, mh[2] = {mn[0], mn[1]};
        if (t + 1 < nt) load_keys(t + 1, jn, mn);
        // The tile's mask (§C.1) as two 32-bit words per query position of
        // the item (bit i of word h = key 32 h + i visible).  Key j (cutoff c)
        // is visible at position q iff j <= q and (j is a sink or
        // q - W - D < max(j, c)): positions lo = j .. hi = max(j, c) + W + D - 1
        // (no end for a sink).  Lane i holds keys i and 32 + i.  A tile whose
        // keys all see every position of the item is only flagged; otherwise,
        // per 32 positions, lane i forms the row of key 32 h + i (bit x =
        // position x of the group visible) and a bit transpose across the
        // warp turns the 32 rows into the 32 positions' words.
        uint32_t* rm = reinterpret_cast<uint32_t*>(meta + st * SM::META_INTS);
        int lo[2], hi[2];
        uint32_t always_b[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          lo[h] = jh[h] >= 0 ? jh[h] : INT_MAX;              // past the candidates: never visible
          hi[h] = (jh[h] < S || mh[h] > INT_MAX - WD) ? INT_MAX : mh[h] + WD - 1;
          always_b[h] = __ballot_sync(0xffffffffu, lo[h] <= q0 && hi[h] >= q1 - 1);
        }
        const bool full_tile = (always_b[0] & always_b[1]) == 0xffffffffu;
        if (mw == 0 && lane == 0) rm[2 * kT2Rows] = full_tile ? 1u : 0u;
        if (!full_tile) {
          // positions in groups of 32, alternating between the two mask warps
          for (int r0 = 32 * mw; r0 < p.qt; r0 += 32 * (kT2Mma - kT2Mask)) {
            const int g0 = q0 + r0;
            uint32_t wd[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int a = lo[h] == INT_MAX ? 32 : max(lo[h] - g0, -1);
              const int b = hi[h] == INT_MAX ? 31 : min(hi[h] - g0, 32);
              wd[h] = warp_transpose32(bit_range32(a, b), lane);
            }
            if (r0 + lane < p.qt) *reinterpret_cast<uint2*>(rm + 2 * (r0 + lane)) = make_uint2(wd[0], wd[1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&meta_full[st]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cand_free[i & 1]);
    }
  } else if (warp >= kT2Mma) {
    // ---------------- MMA issue: one thread per row block ----------------
    // Per block, over the CTA's tiles T of all its items: O += P V(T) once
    // the softmax has written P(T) over S(T) (accumulating unless T is its
    // item's first), and S(T) = Q K(T)^T once its K tile, its item's tile
    // count and Q rows are in and P V(T - 2) has been issued (S(T) reuses
    // that buffer; one thread's MMAs run in issue order).  The thread polls
    // all three conditions, so a P V never waits behind the next item's
    // first S; and it loads the next item's Q rows by TMA as soon as the
    // current item's last S has completed.  The blocks do not wait for each
    // other; a stage is free once both blocks' P V of it completed.
    const int XB = warp - kT2Mma;
    if (lane == 0) {
      const uint32_t qb = sbase + static_cast<uint32_t>(SM::Q_OFF + XB * SM::QBLK);
      // Q rows of block XB of item i: per head one box of PB positions x 64 dims per 64-dim group
      auto load_q = [&](int i) {
        const T2Item w = t2_item(p, ntq, blockIdx.x + i * gridDim.x);
        mbar_arrive_expect_tx(&q_full[XB], static_cast<uint32_t>(SM::QBLK));
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int c = 0; c < SM::NGRP; ++c)
            tma_load_3d(qb + static_cast<uint32_t>(c * SM::QGRP + g * PB * 128), &qmap, 64 * c, w.q0 + XB * PB,
                        w.b * p.Hq + w.hk * G + g, &q_full[XB]);
      };
      // S_X(T) = Q_X K(T)^T: A = Q_X and B = the K tile, both K-major swizzled in shared memory
      auto issue_s = [&](int T) {
        const int st = T % NST;
        const uint32_t kb = sbase + static_cast<uint32_t>(SM::KV_OFF + st * SM::STAGE);
        const uint32_t d = tmem + kColS + static_cast<uint32_t>((2 * XB + (T & 1)) * kT2Keys);
        // 16 dims = 32 bytes of a 128-byte swizzled row; 8-row groups 1024 bytes apart
#pragma unroll
        for (int ks = 0; ks < DH / 16; ++ks)
          tc_mma(d, tc_desc_sw128(qb + static_cast<uint32_t>((ks >> 2) * SM::QGRP + (ks & 3) * 32), 16, 1024),
                 tc_desc_sw128(kb + static_cast<uint32_t>((ks >> 2) * SM::GRP + (ks & 3) * 32), 16, 1024), kIdescS,
                 ks > 0 ? 1u : 0u);
        tc_commit(&s_full[2 * XB + (T & 1)]);
      };
      // O_X (+)= P_X(T) V(T): A = P_X(T) in TMEM over S_X(T) (8 columns per 16 keys), B = the V tile
      auto issue_pv = [&](int T, bool first) {
        const int st = T % NST;
        const uint32_t vb = sbase + static_cast<uint32_t>(SM::KV_OFF + st * SM::STAGE + SM::KV_TILE);
        const uint32_t d = tmem + static_cast<uint32_t>(XB * DH);
        const uint32_t ap = tmem + kColS + static_cast<uint32_t>((2 * XB + (T & 1)) * kT2Keys);
        // MN-major B: 64-dim groups GRP bytes apart (leading), 8-key groups 1024 bytes apart (stride);
        // 16 keys per instruction = two 8-key groups
#pragma unroll
        for (int kk = 0; kk < kT2Keys / 16; ++kk)
          tc_mma_ts(d, ap + 8u * kk, tc_desc_sw128(vb + static_cast<uint32_t>(kk * 2048), SM::GRP, 1024), kIdescPV,
                    (!first || kk > 0) ? 1u : 0u);
        tc_commit(&o_done[XB]);
      };
      // S cursor: item si (tile count snt once known, -1 before), its tile st_; Ts = next S, Tp = next P V
      int si = 0, st_ = 0, snt = -1, Ts = 0, Tp = 0, q_loaded = 0;
      uint32_t first_bits = 0u;   // bit T % 4: tile T is its item's first
      bool more = true;
      load_q(0);
      uint64_t idle_since = 0;
      while (more || Tp < Ts) {
        bool prog = false;
        // the next item's Q, once the item before's last S has read Q
        if (more && q_loaded < si && mbar_test(&q_free[XB], (si - 1) & 1)) {
          load_q(si);
          q_loaded = si;
          prog = true;
        }
        // with no S waiting for its inputs, the thread suspends on the next P
        // (up to ~200 ns a time) instead of spinning on the softmax warps' issue slots
        const bool s_waits = more && Ts < Tp + 2;
        if (Tp < Ts && (s_waits ? mbar_test(&p_full[2 * XB + (Tp & 1)], (Tp >> 1) & 1)
                                : mbar_try_wait_ns(&p_full[2 * XB + (Tp & 1)], (Tp >> 1) & 1, 200u))) {
          tc_fence_after();
          issue_pv(Tp, ((first_bits >> (Tp & 3)) & 1u) != 0u);
          tc_commit(&kv_free[Tp % NST]);
          ++Tp;
          prog = true;
        }
        if (more && Ts < Tp + 2) {
          bool ready = true;
          if (snt < 0) {
            ready = mbar_test(&item_full[si % kT2Ring], (si / kT2Ring) & 1);
            if (ready) {
              snt = ntiles_of(count_ring[si % kT2Ring]);
              st_ = 0;
            }
          }
          // an item's first S waits for its Q rows, and for the item before's
          // last P V to be issued, which the epilogue of that item waits for
          if (ready && st_ == 0) ready = q_loaded == si && (si == 0 || Tp == Ts) && mbar_test(&q_full[XB], si & 1);
          if (ready && mbar_test(&kv_full[Ts % NST], (Ts / NST) & 1)) {
            tc_fence_after();
            issue_s(Ts);
            first_bits = (first_bits & ~(1u << (Ts & 3))) | ((st_ == 0 ? 1u : 0u) << (Ts & 3));
            ++Ts;
            if (++st_ == snt) {
              tc_commit(&q_free[XB]);   // completes once this item's S MMAs have read Q
              ++si;
              snt = -1;
              more = static_cast<int>(blockIdx.x) + si * static_cast<int>(gridDim.x) < nitems;
            }
            prog = true;
          }
        }
        if (prog) {
          idle_since = 0;
        } else {
          if (*abort_flag) break;
          const uint64_t now = global_ns();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            set_error(p.err, DEVERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          if (s_waits || Tp == Ts) __nanosleep(32);   // otherwise the P wait above suspended
        }
      }
    }
    __syncwarp();
  } else {
    // ---------------- softmax: block X, thread = row = TMEM lane ----------------
    const int X = warp >> 2;
    const int row = tid & 127;
    const int posoff = X * PB + row % PB;
    const uint32_t lrow = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tO = tmem + static_cast<uint32_t>(X * DH);
    const bool out32 = (reinterpret_cast<uintptr_t>(p.out) & 31u) == 0u;   // output rows 32-byte aligned
    int T = 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int it = blockIdx.x + i * gridDim.x;
      if (it >= nitems) break;
      if (!__all_sync(0xffffffffu, wait(&item_full[i % kT2Ring], (i / kT2Ring) & 1))) break;
      const T2Item w = t2_item(p, ntq, it);
      const int nt = ntiles_of(count_ring[i % kT2Ring]);
      const int qpos = w.q0 + posoff;
      const bool vrow = qpos < w.q1;
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = 0; t < nt; ++t, ++T) {
        const int st = T % NST;
        bool got = wait(&meta_full[st], (T / NST) & 1);
        got = got && wait(&s_full[2 * X + (T & 1)], (T >> 1) & 1);
        if (!__all_sync(0xffffffffu, got)) {   // the TMEM loads below are warp-collective
          ok = false;
          break;
        }
        tc_fence_after();
        // S(T) row: 64 fp32 columns of buffer T & 1
        const uint32_t tS = tmem + kColS + static_cast<uint32_t>((2 * X + (T & 1)) * kT2Keys);
        static_assert(kT2Keys == 64, "one 64-column TMEM load per tile");
        float sv[kT2Keys];
        tc_ld64(tS + lrow, sv);
        // mask on the raw logits; the tile max commutes with the positive scale,
        // so each weight is one FMA and one ex2: p = 2^(s * scale - m)
        const uint32_t* rmk = reinterpret_cast<const uint32_t*>(meta + st * SM::META_INTS);
        uint32_t vm0 = 0u, vm1 = 0u;
        if (vrow) {
          const bool full = rmk[2 * kT2Rows] != 0u;
          vm0 = full ? 0xffffffffu : rmk[2 * posoff];
          vm1 = full ? 0xffffffffu : rmk[2 * posoff + 1];
        }
        float tmax = -INFINITY;
        if (!__all_sync(0xffffffffu, (vm0 & vm1) == 0xffffffffu)) {
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            sv[x] = ((vm0 >> x) & 1u) ? sv[x] : -INFINITY;
            sv[32 + x] = ((vm1 >> x) & 1u) ? sv[32 + x] : -INFINITY;
          }
        }
        {
          // four independent chains of three-input maxima (chain c: columns c, c + 4, ...), then their max
          float m4[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            m4[c] = fmax3(sv[c], sv[c + 4], sv[c + 8]);
#pragma unroll
            for (int x = c + 12; x < kT2Keys - 4; x += 8) m4[c] = fmax3(m4[c], sv[x], sv[x + 4]);
            m4[c] = fmaxf(m4[c], sv[kT2Keys - 4 + c]);
          }
          tmax = fmax3(fmax3(m4[0], m4[1], m4[2]), m4[3], m4[3]);
        }
        const float tm = tmax * p.scale_log2;
        float alpha = 1.f;
        bool resc = false;
        if (tm > m_run + kT2Lazy) {
          resc = (m_run != -INFINITY);
          alpha = resc ? ex2_approx(m_run - tm) : 0.f;
          l_run *= alpha;
          m_run = tm;
        }
        const float nm = (m_run == -INFINITY) ? 0.f : -m_run;   // masked logits give 2^-inf = 0
        // P(T) in bf16 over the first 32 columns of S(T), 16 columns at a time;
        // the exponent arguments and the row sum on pairs (fp32x2 FMA and add)
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2), nm2 = make_float2(nm, nm);
        float2 ps2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};   // two independent partial sums of pairs
#pragma unroll
        for (int h = 0; h < kT2Keys / 32; ++h) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const float2 xx = __ffma2_rn(make_float2(sv[32 * h + x], sv[32 * h + x + 1]), sc2, nm2);
            const float2 pp = make_float2(ex2_approx(xx.x), ex2_approx(xx.y));
            ps2[(x >> 1) & 1] = __fadd2_rn(ps2[(x >> 1) & 1], pp);
            pk[x / 2] = pack_bf16(pp.x, pp.y);
          }
          tc_st16u(tS + static_cast<uint32_t>(16 * h) + lrow, pk);
        }
        l_run += (ps2[0].x + ps2[1].x) + (ps2[0].y + ps2[1].y);
        if (__any_sync(0xffffffffu, resc)) {
          // rescale this row of O once the P V before (of tile T - 1, same item: t > 0) has completed
          const bool done = wait(&o_done[X], (T - 1) & 1);
          if (!__all_sync(0xffffffffu, done)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = resc ? alpha : 1.f;
#pragma unroll 1
          for (int c0 = 0; c0 < DH; c0 += 32) {
            float o[32];
            tc_ld32(tO + lrow + c0, o);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= f;
            tc_st32(tO + lrow + c0, o);
          }
        }
        // A parity wait on o_done (one phase per P V) is exact only while at
        // most one phase separates it from the barrier's: here P V(T - 2) has
        // completed (S(T) was issued after it) and P V(T) waits for this
        // arrival.  So the item's last tile waits here for P V(T - 1), and the
        // epilogue then waits for P V(T) alone.
        if (t == nt - 1 && t > 0 && !__all_sync(0xffffffffu, wait(&o_done[X], (T - 1) & 1))) {
          ok = false;
          break;
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&p_full[2 * X + (T & 1)]);
      }
      if (!ok) break;
      // epilogue: O of this row once the item's last P V (tile T - 1) has completed; the
      // next item's first P V overwrites O only after this thread's next p_full arrival
      if (!__all_sync(0xffffffffu, wait(&o_done[X], (T - 1) & 1))) break;
      tc_fence_after();
      const size_t rowi = (static_cast<size_t>(w.b) * p.Hq + w.hk * G + row / PB) * n + (vrow ? qpos : 0);
      __nv_bfloat16* og = static_cast<__nv_bfloat16*>(p.out) + rowi * DH;
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < DH; c0 += 64) {
        float o[64];
        tc_ld64(tO + lrow + c0, o);
        if (vrow) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(o[2 * c] * inv, o[2 * c + 1] * inv);
          if (out32) {   // one full 32-byte sector per store
#pragma unroll
            for (int c = 0; c < 4; ++c) st_global_v8(og + c0 + 16 * c, pk + 8 * c);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(og + c0 + 8 * c) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
      }
      if (vrow && p.lse != nullptr) p.lse[rowi] = (m_run + log2f(l_run)) * 0.69314718055994531f;
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kT2Mma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem), "r"(kT2Cols) : "memory");
  }
}

// The driver's tensor-map encoder, fetched through the runtime (no link-time
// dependency on libcuda); null if unavailable.
PFN_cuTensorMapEncodeTiled_v12000 attn_tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) != cudaSuccess ||
        qres != cudaDriverEntryPointSuccess || fn == nullptr)
      return nullptr;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  return encode;
}

// One CTA per SM (at most one per work item); Q through a 3-D tensor map
// (head dim, position, batch row x query head) with one box per head and
// 64-dim group.
template <int DH, int NST>
int launch_attn_tcp_stages(const PaArgs& pa, int units, int n, size_t smem, cudaStream_t st) {
  if (cudaFuncSetAttribute(sparse_attn_tcp_kernel<DH, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return -1;
  PFN_cuTensorMapEncodeTiled_v12000 encode = attn_tensor_map_encoder();
  if (encode == nullptr) return -1;
  const int B = units / pa.Hkv;
  CUtensorMap qmap;
  const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(DH), static_cast<cuuint64_t>(n),
                              static_cast<cuuint64_t>(B) * pa.Hq};
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(DH) * 2, static_cast<cuuint64_t>(n) * DH * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(128 / pa.G), 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  if (encode(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(pa.q), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return -1;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return -1;
  const int64_t nitems = static_cast<int64_t>(units) * ((n + pa.qt - 1) / pa.qt);
  if (nitems > (1ll << 30)) return -2;
  const int grid = static_cast<int>(nitems < nsm ? nitems : nsm);
  sparse_attn_tcp_kernel<DH, NST><<<grid, kT2Threads, smem, st>>>(qmap, pa, static_cast<int>(nitems));
  return 0;
}

// Four stages when they fit in shared memory beside the candidate lists, else three.
template <int DH>
int launch_attn_tcp(const PaArgs& pa, int units, int n, cudaStream_t st) {
  constexpr size_t kMax = 227 * 1024;
  if (units == 0 || n == 0) return 0;
  if (pa.G > 16 || 128 % pa.G != 0) return -2;   // one TMA box of at least 8 rows per head
  const size_t smem4 = T2Smem<DH, 4>::bytes(pa.cand_cap);
  if (smem4 <= kMax) return launch_attn_tcp_stages<DH, 4>(pa, units, n, smem4, st);
  const size_t smem3 = T2Smem<DH, 3>::bytes(pa.cand_cap);
  if (smem3 <= kMax) return launch_attn_tcp_stages<DH, 3>(pa, units, n, smem3, st);
  return -2;
}

template <int DH>
int launch_attn_f32(const PaArgs& pa, int units, int n, cudaStream_t st) {
  const size_t smem = PaSmem<DH>::bytes(pa.cand_cap);
  // set on every call: the attribute belongs to the current device
  if (smem > 48 * 1024 && cudaFuncSetAttribute(sparse_attn_kernel<float, DH>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem)) != cudaSuccess)
    return -1;
  dim3 grid((n + pa.qt - 1) / pa.qt, units);
  sparse_attn_kernel<float, DH><<<grid, kPaThreads, smem, st>>>(pa);
  return 0;
}

// ---------------- cache build from the cutoffs ----------------
// Long-range set at the last prompt position = the tokens whose cutoff is
// "never"; a whole-prompt prefill places them in ascending position order.
__global__ void __launch_bounds__(256) place_kept_kernel(LayerArgs a, const int32_t* __restrict__ cut,
                                                         const float* __restrict__ scores, int score_cap, int n,
                                                         int ne, const uint8_t* __restrict__ k,
                                                         const uint8_t* __restrict__ v, int half) {
  __shared__ int wtot[8];
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t* cu = cut + static_cast<size_t>(u) * n;
  const int base_slot = a.S + a.W + a.D;
  int count = 0;
  for (int b0 = 0; b0 < ne; b0 += 256) {
    const int i = b0 + tid;
    const int j = a.S + i;
    const bool f = i < ne && cu[j] == kNever;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wtot[warp] = __popc(bal);
    __syncthreads();
    int off = count, total = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      off += (w < warp) ? wtot[w] : 0;
      total += wtot[w];
    }
    off += __popc(bal & ((1u << lane) - 1u));
    if (f && off < a.K) {
      const int slot = base_slot + off;
      uint8_t* dst = a.kv + (static_cast<size_t>(u) * a.NS + slot) * a.row_bytes;
      const uint8_t* ks = k + (static_cast<size_t>(u) * n + j) * half;
      const uint8_t* vs = v + (static_cast<size_t>(u) * n + j) * half;
      for (int b = 0; b < half; b += 16) {
        *reinterpret_cast<uint4*>(dst + b) = *reinterpret_cast<const uint4*>(ks + b);
        *reinterpret_cast<uint4*>(dst + half + b) = *reinterpret_cast<const uint4*>(vs + b);
      }
      a.pos[static_cast<size_t>(u) * a.NS + slot] = j;
      a.score[static_cast<size_t>(u) * a.NS + slot] = scores[static_cast<size_t>(u) * score_cap + i];
    }
    count += total;
    __syncthreads();
  }
  if ((a.flags & FLAG_DEBUG_CHECKS) && tid == 0 && count != min(a.K, ne)) set_error(a.err, DEVERR_STATE_MISMATCH);
}

}  // namespace

int launch_place_kept(const LayerArgs& a, int dtype, const PrefillAttnPlan& p, const void* k, const void* v,
                      const uint8_t* workspace, cudaStream_t st) {
  if (p.ne <= 0 || a.K <= 0) return 0;
  const int half = a.d * (dtype == 0 ? 4 : 2);
  place_kept_kernel<<<a.units, 256, 0, st>>>(a, reinterpret_cast<const int32_t*>(workspace + p.cut_off),
                                             reinterpret_cast<const float*>(workspace + p.score_off), p.ne, p.n,
                                             p.ne, static_cast<const uint8_t*>(k), static_cast<const uint8_t*>(v),
                                             half);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int plan_prefill_attention(const LayerArgs& a, int dtype, int n, PrefillAttnPlan* p) {
  if (n < 0 || kPaRows % a.G != 0) return -2;
  if (dtype != 0 && a.G > 16) return -2;   // bf16: each head's rows of a row block are one TMA box of >= 8 rows (a cache has G <= 8)
  if (a.mlstm) return -2;   // the prompt scores come from the stateless scorers or the caller
  if (a.d != 64 && a.d != 128) return -2;
  PrefillAttnPlan P{};
  P.n = n;
  P.ne = max(0, n - a.W - a.D - a.S);
  P.npow = next_pow2(max(P.ne, 1));
  P.words = max(1, (P.ne + 31) / 32);
  P.qt = (dtype == 0 ? kPaRows : kT2Rows) / a.G;
  const int64_t cc = static_cast<int64_t>(a.S) + a.K + P.qt + a.W + a.D;
  if (cc > (1 << 14)) return -2;   // the candidate list lives in shared memory
  P.cand_cap = static_cast<int>(cc);
  P.keys_global = P.npow > kPaSmemSortKeys;
  P.bits_global = P.words > kPaSmemBitmapWords;
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t units = a.units;
  size_t off = 0;
  P.cut_off = off;
  off += al(units * max(n, 1) * sizeof(int32_t));
  P.score_off = off;
  off += al(units * max(P.ne, 1) * sizeof(float));
  P.order_off = off;
  off += al(units * max(P.ne, 1) * sizeof(int32_t));
  P.keys_off = off;
  if (P.keys_global) off += al(units * P.npow * sizeof(uint64_t));
  P.bits_off = off;
  if (P.bits_global) off += al(units * P.words * sizeof(uint32_t));
  P.total = max(off, static_cast<size_t>(256));
  *p = P;
  return 0;
}

int launch_prefill_attention(const LayerArgs& a, int dtype, const PrefillAttnPlan& p, const void* q, const void* k,
                             const void* v, const float* ext, void* out, float* lse, uint8_t* workspace,
                             cudaStream_t st, bool reuse_cutoffs) {
  if (p.n == 0) return 0;
  if (a.units > 65535) return -2;
  int32_t* cut = reinterpret_cast<int32_t*>(workspace + p.cut_off);
  float* scores = reinterpret_cast<float*>(workspace + p.score_off);
  uint64_t* keys = reinterpret_cast<uint64_t*>(workspace + p.keys_off);
  uint32_t* bits = reinterpret_cast<uint32_t*>(workspace + p.bits_off);
  int32_t* order = reinterpret_cast<int32_t*>(workspace + p.order_off);
  if (!reuse_cutoffs && p.ne > 0) {
    const int r = launch_prompt_scores(a, dtype, k, v, p.n, ext, scores, p.ne, st);
    if (r != 0) return r;
  }
  if (!reuse_cutoffs) {
    const size_t cut_smem = p.keys_global ? 0 : static_cast<size_t>(p.npow) * 8;
    if (cudaFuncSetAttribute(cutoff_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPaSmemSortKeys * 8) !=
        cudaSuccess)
      return -1;
    cutoff_kernel<<<a.units, kCutThreads, cut_smem, st>>>(scores, max(p.ne, 1), cut, order, p.n, p.ne, p.npow, a.S,
                                                          keys, p.keys_global ? 1 : 0);
    const size_t walk_smem = p.bits_global ? 0 : static_cast<size_t>(kWalkWarps) * p.words * 4;
    if (cudaFuncSetAttribute(walk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kWalkWarps * kPaSmemBitmapWords * 4) != cudaSuccess)
      return -1;
    walk_kernel<<<(a.units + kWalkWarps - 1) / kWalkWarps, 32 * kWalkWarps, walk_smem, st>>>(
        order, cut, p.n, p.ne, p.words, a.S, a.K, a.units, bits, p.bits_global ? 1 : 0, a.err);
  }
  PaArgs pa;
  pa.q = q;
  pa.k = k;
  pa.v = v;
  pa.out = out;
  pa.lse = lse;
  pa.cut = cut;
  pa.n = p.n;
  pa.S = a.S;
  pa.W = a.W;
  pa.D = a.D;
  pa.G = a.G;
  pa.Hq = a.Hq;
  pa.Hkv = a.Hkv;
  pa.qt = p.qt;
  pa.cand_cap = p.cand_cap;
  pa.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d));
  pa.err = a.err;
  int r;
  if (dtype == 0)
    r = (a.d == 128) ? launch_attn_f32<128>(pa, a.units, p.n, st) : launch_attn_f32<64>(pa, a.units, p.n, st);
  else
    r = (a.d == 128) ? launch_attn_tcp<128>(pa, a.units, p.n, st) : launch_attn_tcp<64>(pa, a.units, p.n, st);
  if (r != 0) return r;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kvpop
