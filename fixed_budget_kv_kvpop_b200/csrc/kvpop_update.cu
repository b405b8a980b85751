// Fused boundary update of one decode step (KVpop page §3 Fixed-budget pruning,
// §C.1 Mask Definition, §E.4 Delayed Readout, §I Pseudocode).
//
// Per (batch row, KV head) unit, with p = the new token's position:
//   1. the token o = p - W leaves the window; with a staging ring (D > 0) it
//      moves to staging slot S + W + (o mod D) and the staged token b = o - D
//      reaches the eviction boundary; with D = 0, b = o;
//   2. b is scored: s = w2 . relu(W1 [k_b; v_b] + b1) + b2 (fp64 accumulation,
//      rounded to fp32, the ranking precision), or the
//      caller's score stored when b arrived;
//   3. while fewer than K long-range slots are used, b takes the next free one;
//      otherwise the slot m holding the minimum key (score, -position) is found
//      by a block argmin and b replaces it in place only if key(b) > key(m);
//   4. the new token's k/v is written to its window (or sink) slot.
// One CTA per unit; all steps are ordered inside the CTA with __syncthreads.
#include "kvpop_internal.cuh"

namespace kvpop {

namespace {

constexpr int kUpdThreads = 128;

template <typename T>
__device__ __forceinline__ void copy_row(uint8_t* dst, const uint8_t* src, int bytes) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
  for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) d[i] = s[i];
}

template <typename T>
__global__ void __launch_bounds__(kUpdThreads) update_kernel(LayerArgs a, const T* __restrict__ k_new,
                                                             const T* __restrict__ v_new,
                                                             const float* __restrict__ ext_score) {
  extern __shared__ double smem_d[];
  double* red = smem_d;                               // 32 doubles
  float* xs = reinterpret_cast<float*>(smem_d + 32);  // 2d floats
  __shared__ unsigned long long s_min_key[kUpdThreads / 32];
  __shared__ int s_min_slot[kUpdThreads / 32];
  __shared__ int s_decision[2];     // target slot, admit

  const int u = blockIdx.x;
  const int h = u % a.Hkv;
  const int tid = threadIdx.x;
  const int S = a.S, W = a.W, D = a.D, K = a.K, NS = a.NS;
  int32_t* st = a.state + 4 * u;
  const int p = st[0];
  const int n_topk = st[1];
  if (p >= a.max_context) {
    if (tid == 0) set_error(a.err, DEVERR_CONTEXT_OVERFLOW);
    return;
  }
  uint8_t* kv = a.kv + static_cast<size_t>(u) * NS * a.row_bytes;
  int32_t* pos = a.pos + static_cast<size_t>(u) * NS;
  float* score = a.score + static_cast<size_t>(u) * NS;
  const bool ext = (a.flags & FLAG_EXTERNAL_SCORES) != 0;

  const int ns = p < S ? p : window_slot(p, S, W);
  const int o = (p >= S && p - W >= S) ? p - W : -1;
  int bpos, bslot, st_slot = -1;
  if (D > 0) {
    st_slot = o >= 0 ? staging_slot(o, S, W, D) : -1;
    bpos = (o >= 0 && o - D >= S) ? o - D : -1;
    bslot = st_slot;
  } else {
    bpos = o;
    bslot = ns;
  }
  const int base = topk_base(S, W, D);

  if (bpos >= 0) {
    const uint8_t* brow = kv + static_cast<size_t>(bslot) * a.row_bytes;
    float sb;
    if (ext) {
      sb = score[bslot];
    } else {
      sb = mlp_score_block<T>(reinterpret_cast<const T*>(brow), a.d,
                              a.w1 + static_cast<size_t>(h) * a.hidden * 2 * a.d,
                              a.b1 + static_cast<size_t>(h) * a.hidden, a.w2 + static_cast<size_t>(h) * a.hidden,
                              a.b2[h], a.hidden, xs, red);
    }
    if ((a.flags & FLAG_DEBUG_CHECKS) && tid == 0) {
      if (pos[bslot] != bpos) set_error(a.err, DEVERR_STATE_MISMATCH);
      if (sb != sb) set_error(a.err, DEVERR_NAN_SCORE);
    }
    int target = -1;
    if (n_topk < K) {
      target = base + n_topk;
    } else if (K > 0) {
      // block argmin of rank keys over the K long-range slots
      unsigned long long best = ~0ull;
      int best_slot = -1;
      for (int i = tid; i < K; i += blockDim.x) {
        unsigned long long key = rank_key(score[base + i], pos[base + i]);
        if (key < best) { best = key; best_slot = base + i; }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        unsigned long long ok = __shfl_xor_sync(0xffffffffu, best, off);
        int os = __shfl_xor_sync(0xffffffffu, best_slot, off);
        if (ok < best) { best = ok; best_slot = os; }
      }
      if ((tid & 31) == 0) { s_min_key[tid >> 5] = best; s_min_slot[tid >> 5] = best_slot; }
      __syncthreads();
      if (tid == 0) {
        unsigned long long b = s_min_key[0];
        int bs = s_min_slot[0];
        for (int w = 1; w < kUpdThreads / 32; ++w)
          if (s_min_key[w] < b) { b = s_min_key[w]; bs = s_min_slot[w]; }
        s_decision[0] = (rank_key(sb, bpos) > b) ? bs : -1;
      }
      __syncthreads();
      target = s_decision[0];
    }
    if (target >= 0) {
      copy_row<T>(kv + static_cast<size_t>(target) * a.row_bytes, brow, a.row_bytes);
      if (tid == 0) { score[target] = sb; pos[target] = bpos; }
    }
    __syncthreads();
  }
  if (D > 0 && o >= 0) {
    copy_row<T>(kv + static_cast<size_t>(st_slot) * a.row_bytes, kv + static_cast<size_t>(ns) * a.row_bytes,
                a.row_bytes);
    if (tid == 0) { pos[st_slot] = o; score[st_slot] = score[ns]; }
    __syncthreads();
  }
  // new token -> its window (or sink) slot
  {
    T* dst = reinterpret_cast<T*>(kv + static_cast<size_t>(ns) * a.row_bytes);
    const T* kn = k_new + static_cast<size_t>(u) * a.d;
    const T* vn = v_new + static_cast<size_t>(u) * a.d;
    for (int i = tid; i < a.d; i += blockDim.x) { dst[i] = kn[i]; dst[a.d + i] = vn[i]; }
    if (tid == 0) {
      pos[ns] = p;
      score[ns] = ext ? ext_score[u] : 0.f;
      st[0] = p + 1;
      st[1] = (bpos >= 0 && n_topk < K) ? n_topk + 1 : n_topk;
    }
  }
}

}  // namespace

int launch_update(const LayerArgs& a, int dtype, const void* k_new, const void* v_new, const float* ext_score,
                  cudaStream_t st) {
  const size_t smem = 32 * sizeof(double) + 2 * a.d * sizeof(float);
  if (dtype == 0) {
    update_kernel<float><<<a.units, kUpdThreads, smem, st>>>(a, static_cast<const float*>(k_new),
                                                            static_cast<const float*>(v_new), ext_score);
  } else {
    update_kernel<__nv_bfloat16><<<a.units, kUpdThreads, smem, st>>>(
        a, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new), ext_score);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kvpop
