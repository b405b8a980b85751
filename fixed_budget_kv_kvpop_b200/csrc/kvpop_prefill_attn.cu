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
// masking each (query, key) pair by the rule above.
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

// ---------------- cutoffs: one CTA per unit ----------------
__global__ void __launch_bounds__(kCutThreads) cutoff_kernel(const float* __restrict__ scores, int score_cap,
                                                             int32_t* __restrict__ cut, int n, int ne, int npow,
                                                             int words, int S, int K, uint64_t* keys_g,
                                                             uint32_t* bits_g, int keys_global, int bits_global,
                                                             int32_t* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  int32_t* cu = cut + static_cast<size_t>(u) * n;
  uint64_t* keys = keys_global ? keys_g + static_cast<size_t>(u) * npow : reinterpret_cast<uint64_t*>(smem_raw);
  uint32_t* bits = bits_global ? bits_g + static_cast<size_t>(u) * words
                               : reinterpret_cast<uint32_t*>(smem_raw + (keys_global ? 0 : static_cast<size_t>(npow) * 8));
  // tokens that never become eligible in the prompt
  for (int t = tid; t < n; t += blockDim.x)
    if (t < S || t >= S + ne) cu[t] = -1;
  if (ne == 0) return;
  const float* su = scores + static_cast<size_t>(u) * score_cap;
  for (int i = tid; i < npow; i += blockDim.x) keys[i] = (i < ne) ? rank_key(su[i], S + i) : 0ull;
  for (int i = tid; i < words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  // bitonic sort, descending (best first); padding keys (0) sink to the end
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
  if (tid != 0) return;
  // best-first walk; T = K-th smallest position among the tokens seen so far
  int T = -1;
  bool bad = false;
  for (int r = 0; r < ne; ++r) {
    const int pos = static_cast<int>(0xffffffffu - static_cast<uint32_t>(keys[r]));
    int c;
    if (K == 0) {
      c = pos;
    } else if (r < K) {
      c = kNever;
      T = max(T, pos);
      const int idx = pos - S;
      bits[idx >> 5] |= 1u << (idx & 31);
    } else {
      c = max(pos, T);
      if (pos < T) {
        const int idx = pos - S;
        bits[idx >> 5] |= 1u << (idx & 31);
        const int ti = T - S;
        int w = ti >> 5;
        uint32_t m = bits[w] & ((1u << (ti & 31)) - 1u);
        while (m == 0u && w > 0) m = bits[--w];
        if (m == 0u) {  // cannot happen: pos < T was just inserted
          bad = true;
          break;
        }
        T = S + (w << 5) + 31 - __clz(m);
      }
    }
    cu[pos] = c;
  }
  if (bad) set_error(err, DEVERR_STATE_MISMATCH);
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
template <> struct PaIo<__nv_bfloat16> {
  static __device__ __forceinline__ void load8(const __nv_bfloat16* p, float* o) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 r;
    r.x = *reinterpret_cast<const uint32_t*>(&a);
    r.y = *reinterpret_cast<const uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = r;
  }
};

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

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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

  // candidate keys: sinks, long-range tokens kept at the first query, recent block
  const int m0 = q0 - WD;
  const int ns = min(S, q1);
  for (int i = tid; i < ns; i += kPaThreads) cand[i] = i;
  int count = ns;
  for (int base = S; base <= m0; base += kPaThreads) {
    const int j = base + tid;
    const bool f = j <= m0 && cu[j] > m0;
    const unsigned bal = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wtot[warp] = __popc(bal);
    __syncthreads();
    int off = count, total = 0;
#pragma unroll
    for (int w = 0; w < kPaThreads / 32; ++w) {
      const int t = wtot[w];
      off += (w < warp) ? t : 0;
      total += t;
    }
    const int slot = off + __popc(bal & ((1u << lane) - 1u));
    if (f && slot < p.cand_cap) cand[slot] = j;
    count += total;
    __syncthreads();
  }
  const int r0 = max(S, m0 + 1);
  const int nr = max(0, q1 - r0);
  for (int i = tid; i < nr; i += kPaThreads)
    if (count + i < p.cand_cap) cand[count + i] = r0 + i;
  count += nr;
  if (count > p.cand_cap) count = p.cand_cap;   // cannot happen: S + K + qt + W + D bounds it
  __syncthreads();

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

template <typename T, int DH>
int launch_attn(const PaArgs& pa, int units, int n, cudaStream_t st) {
  const size_t smem = PaSmem<DH>::bytes(pa.cand_cap);
  static size_t smem_set = 0;
  if (smem > 48 * 1024 && smem > smem_set) {
    if (cudaFuncSetAttribute(sparse_attn_kernel<T, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -1;
    smem_set = smem;
  }
  dim3 grid((n + pa.qt - 1) / pa.qt, units);
  sparse_attn_kernel<T, DH><<<grid, kPaThreads, smem, st>>>(pa);
  return 0;
}

}  // namespace

int plan_prefill_attention(const LayerArgs& a, int n, PrefillAttnPlan* p) {
  if (n < 0 || kPaRows % a.G != 0) return -2;
  if (a.d != 64 && a.d != 128) return -2;
  PrefillAttnPlan P{};
  P.n = n;
  P.ne = max(0, n - a.W - a.D - a.S);
  P.npow = next_pow2(max(P.ne, 1));
  P.words = max(1, (P.ne + 31) / 32);
  P.qt = kPaRows / a.G;
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
                             cudaStream_t st) {
  if (p.n == 0) return 0;
  if (a.units > 65535) return -2;
  int32_t* cut = reinterpret_cast<int32_t*>(workspace + p.cut_off);
  float* scores = reinterpret_cast<float*>(workspace + p.score_off);
  uint64_t* keys = reinterpret_cast<uint64_t*>(workspace + p.keys_off);
  uint32_t* bits = reinterpret_cast<uint32_t*>(workspace + p.bits_off);
  if (p.ne > 0) {
    const int r = launch_prompt_scores(a, dtype, k, v, p.n, ext, scores, p.ne, st);
    if (r != 0) return r;
  }
  const size_t cut_smem = (p.keys_global ? 0 : static_cast<size_t>(p.npow) * 8) +
                          (p.bits_global ? 0 : static_cast<size_t>(p.words) * 4);
  static bool cut_attr = false;
  if (!cut_attr) {
    const int mx = kPaSmemSortKeys * 8 + kPaSmemBitmapWords * 4;
    if (cudaFuncSetAttribute(cutoff_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess)
      return -1;
    cut_attr = true;
  }
  cutoff_kernel<<<a.units, kCutThreads, cut_smem, st>>>(scores, max(p.ne, 1), cut, p.n, p.ne, p.npow, p.words, a.S,
                                                        a.K, keys, bits, p.keys_global ? 1 : 0,
                                                        p.bits_global ? 1 : 0, a.err);
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
  int r;
  if (dtype == 0)
    r = (a.d == 128) ? launch_attn<float, 128>(pa, a.units, p.n, st) : launch_attn<float, 64>(pa, a.units, p.n, st);
  else
    r = (a.d == 128) ? launch_attn<__nv_bfloat16, 128>(pa, a.units, p.n, st)
                     : launch_attn<__nv_bfloat16, 64>(pa, a.units, p.n, st);
  if (r != 0) return r;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kvpop
