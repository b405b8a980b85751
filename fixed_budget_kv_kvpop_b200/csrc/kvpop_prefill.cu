// Prefill builder: appends a chunk of prompt tokens to the KVpop cache.
//
// After a chunk the cache holds exactly what the running prefix top-k rule
// (KVpop page §I Pseudocode, §C.1 Mask Definition) gives at the chunk's last
// token: positions < S in the sink slots, the last W tokens in the window
// ring, the D tokens before them in the staging ring, and the K best tokens
// (key = (score, -position), fp32 scores as in §F) among all tokens that have
// left the window/staging, in the long-range slots.
//
// Placement: long-range tokens that survive the chunk keep their slots; the
// admitted newcomers, in ascending position, take the free-or-vacated
// long-range slots in ascending slot order (for a first chunk this is
// ascending position order).
//
// Kernels, in stream order:
//   P1 score:  MLP score of every newly eligible token (or caller's score),
//              as a small register-blocked GEMM with W1 held in smem, fp64
//              accumulation rounded once to fp32.
//   P2 select: per unit, radix select of the K-th largest 64-bit key among the
//              current long-range tokens and the newcomers, then slot
//              assignment by block prefix sums and row copies.
//   P3 move:   window tokens that enter the staging ring move there.
//   P4 write:  chunk tokens go to their sink / window / staging slots.
#include <type_traits>

#include "kvpop_internal.cuh"
#include "kvpop_prefill_attn.cuh"

namespace kvpop {

namespace {

struct ChunkGeom {
  int n0, n1, e0, e1, c0;  // tokens before/after, newly eligible [e0, e1), long-range used before
};

// Where does token t's row live during this chunk?  (t < n0: cache ring)
template <typename T>
__device__ __forceinline__ const uint8_t* token_row(const LayerArgs& a, const ChunkGeom& cg, int u, int t,
                                                    const T* k, const T* v, int n, const uint8_t*& vsrc) {
  if (t >= cg.n0) {
    const size_t off = (static_cast<size_t>(u) * n + (t - cg.n0)) * a.d;
    vsrc = reinterpret_cast<const uint8_t*>(v + off);
    return reinterpret_cast<const uint8_t*>(k + off);
  }
  const int slot = (t >= cg.n0 - a.W) ? window_slot(t, a.S, a.W) : staging_slot(t, a.S, a.W, a.D);
  const uint8_t* row = a.kv + (static_cast<size_t>(u) * a.NS + slot) * a.row_bytes;
  vsrc = row + a.d * sizeof(T);
  return row;
}

template <typename T>
__device__ __forceinline__ int token_slot_in_cache(const LayerArgs& a, const ChunkGeom& cg, int t) {
  return (t >= cg.n0 - a.W) ? window_slot(t, a.S, a.W) : staging_slot(t, a.S, a.W, a.D);
}

// ---------------- P1: scoring ----------------
constexpr int kScoreThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(LayerArgs a, ChunkGeom cg, const T* __restrict__ k,
                                                              const T* __restrict__ v, int n,
                                                              const float* __restrict__ ext,
                                                              float* __restrict__ out, int cap) {
  extern __shared__ float sm[];
  const int u = blockIdx.y;
  const int h = u % a.Hkv;
  const int n_new = cg.e1 - cg.e0;
  const int d2 = 2 * a.d;
  const int HQ = a.hidden / 4;                 // threads per token quad
  const int TT = 4 * (kScoreThreads / HQ);     // tokens per tile
  const int tok0 = blockIdx.x * TT;
  if (tok0 >= n_new) return;
  const int ntok = min(TT, n_new - tok0);
  const int tid = threadIdx.x;

  if (a.flags & FLAG_EXTERNAL_SCORES) {
    for (int i = tid; i < ntok; i += blockDim.x) {
      const int t = cg.e0 + tok0 + i;
      float s;
      if (t >= cg.n0) s = ext[static_cast<size_t>(u) * n + (t - cg.n0)];
      else s = a.score[static_cast<size_t>(u) * a.NS + token_slot_in_cache<T>(a, cg, t)];
      out[static_cast<size_t>(u) * cap + tok0 + i] = ranking_priority(a, u, t + a.W + a.D, s);
    }
    return;
  }

  float* Ws = sm;                          // [d2][hidden]  (W1 transposed)
  float* Xs = sm + d2 * a.hidden;          // [TT][d2]
  const float* w1 = a.w1 + static_cast<size_t>(h) * a.hidden * d2;
  for (int idx = tid; idx < a.hidden * d2; idx += blockDim.x) {
    const int j = idx / d2, i = idx % d2;
    Ws[i * a.hidden + j] = w1[idx];
  }
  for (int idx = tid; idx < TT * d2; idx += blockDim.x) {
    const int tt = idx / d2, i = idx % d2;
    float x = 0.f;
    if (tt < ntok) {
      const int t = cg.e0 + tok0 + tt;
      const uint8_t* vs;
      const uint8_t* ks = token_row<T>(a, cg, u, t, k, v, n, vs);
      x = (i < a.d) ? Elem<T>::to_f32(reinterpret_cast<const T*>(ks)[i])
                    : Elem<T>::to_f32(reinterpret_cast<const T*>(vs)[i - a.d]);
    }
    Xs[tt * d2 + i] = x;
  }
  __syncthreads();
  const int tq = tid / HQ, hq = tid % HQ;
  // fp64 accumulation, one rounding to fp32 at the end (ranking precision)
  double acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0;
  for (int i = 0; i < d2; ++i) {
    const float4 wv = *reinterpret_cast<const float4*>(Ws + i * a.hidden + 4 * hq);
    const double w0 = wv.x, w1v = wv.y, w2v = wv.z, w3 = wv.w;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const double xv = Xs[(4 * tq + r) * d2 + i];
      acc[r][0] = fma(xv, w0, acc[r][0]);
      acc[r][1] = fma(xv, w1v, acc[r][1]);
      acc[r][2] = fma(xv, w2v, acc[r][2]);
      acc[r][3] = fma(xv, w3, acc[r][3]);
    }
  }
  const float* b1 = a.b1 + static_cast<size_t>(h) * a.hidden;
  const float* w2 = a.w2 + static_cast<size_t>(h) * a.hidden;
  double part[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    part[r] = 0.0;
#pragma unroll
    for (int c = 0; c < 4; ++c)
      part[r] = fma(static_cast<double>(w2[4 * hq + c]),
                    fmax(acc[r][c] + static_cast<double>(b1[4 * hq + c]), 0.0), part[r]);
  }
  // reduce over the HQ threads of a token quad (consecutive lanes, HQ | 32)
  for (int off = 1; off < HQ; off <<= 1)
#pragma unroll
    for (int r = 0; r < 4; ++r) part[r] += __shfl_xor_sync(0xffffffffu, part[r], off);
  if (hq == 0) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int tt = 4 * tq + r;
      if (tt < ntok)
        out[static_cast<size_t>(u) * cap + tok0 + tt] =
            ranking_priority(a, u, cg.e0 + tok0 + tt + a.W + a.D, static_cast<float>(part[r] + static_cast<double>(a.b2[h])));
    }
  }
}

// P1 for the common shapes (2d in {128, 256}, hidden in {32, 64}): the same
// scores as score_kernel, with the pre-activations W1 x on the fp64 tensor
// cores (mma.sync m8n8k4 f64: fp64 products and sums, as score_kernel's fp64
// FMAs).  Shared memory holds W1 transposed and a tile of TT tokens' inputs
// [k; v], both in fp32 (exact for fp32 weights and bf16/fp32 inputs; each
// operand fragment is widened to fp64 as it is loaded), with row pitches
// that make every fragment load conflict-free.  Warp w owns tokens 32 (w % 4)
// .. + 31 of the tile (4 row tiles of 8) x part w / 4 of HS equal parts of
// the hidden units: per 4 inputs it loads 4 + HID / (8 HS) fragments and
// issues 4 HID / (8 HS) MMAs; HS warps per scheduler hide each other's MMA
// latency.  The epilogue forms w2 . relu(. + b1) over the warp's part per
// token, sums the 4 lanes of each row by shuffles and the HS parts in a
// fixed order through shared memory.  Each block keeps W1 resident and walks
// tpb consecutive token tiles of its unit (score64_tiles_per_block).
constexpr int kScore64Threads = 512;
constexpr int kScore64Parts = kScore64Threads / 128;   // HS: hidden parts, one warp each per token group

// Tiles per block: the split of each unit's tiles into blocks that
// minimises (waves of one-block-per-SM) x (tiles per block + the cost of a
// block's start, about 0.15 of a tile: W1 and the first tile's rows).
inline int score64_tiles_per_block(int tiles, int units, int nsm) {
  if (tiles <= 0) return 1;
  int best = tiles;
  double best_cost = 1e300;
  for (int c = 1; c <= tiles; ++c) {
    const int tpb = (tiles + c - 1) / c;
    if (c > 1 && tpb == (tiles + c - 2) / (c - 1)) continue;   // same split as c - 1
    const long long blocks = static_cast<long long>(units) * ((tiles + tpb - 1) / tpb);
    const double cost = static_cast<double>((blocks + nsm - 1) / nsm) * (tpb + 0.15);
    if (cost < best_cost) { best_cost = cost; best = tpb; }
  }
  return best;
}

template <int D2, int HID>
struct Score64Geom {
  static constexpr int TT = 128;                               // tokens per tile: 32 per warp pair
  static constexpr int XP = D2 + 4;                            // floats per token row (pitch = 4 mod 32)
  static constexpr int WP = HID + 8;                           // floats per input row of W1^T (pitch = 8 mod 32)
  static constexpr int SMEM = (D2 * WP + TT * XP) * 4 + kScore64Parts * TT * 8;   // + the parts' partial sums
};

__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1]) : "d"(a), "d"(b));
}

template <typename T, int D2, int HID>
__global__ void __launch_bounds__(kScore64Threads, 1) score64_kernel(LayerArgs a, ChunkGeom cg,
                                                                     const T* __restrict__ k,
                                                                     const T* __restrict__ v, int n,
                                                                     float* __restrict__ out, int cap, int tpb) {
  using SG = Score64Geom<D2, HID>;
  constexpr int TT = SG::TT, XP = SG::XP, WP = SG::WP;
  constexpr int HS = kScore64Parts;
  constexpr int NT = HID / (8 * HS);                            // column tiles of this warp's hidden part
  static_assert(NT >= 1 && HID % (8 * HS) == 0, "whole column tiles per part");
  constexpr int EPU = 16 / static_cast<int>(sizeof(T));        // inputs per 16-byte load
  constexpr int UPT = D2 / EPU;                                 // 16-byte loads per token row
  extern __shared__ __align__(16) float smf[];
  float* Wt = smf;                                              // [D2][WP]: Wt[i][j] = W1[j][i]
  float* Xs = smf + D2 * WP;                                    // [TT][XP]: Xs[t][i] = x_t[i]
  double* pp = reinterpret_cast<double*>(Xs + TT * XP);         // [part][TT] partial sums
  const int u = blockIdx.y;
  const int h = u % a.Hkv;
  const int n_new = cg.e1 - cg.e0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile0 = blockIdx.x * tpb;
  if (tile0 * TT >= n_new) return;

  {
    // W1 [HID][D2] -> Wt: thread -> hidden j = e % HID, inputs 4 q .. 4 q + 3
    // with q = e / HID (consecutive lanes write consecutive j of one input
    // row), all of a thread's loads in flight before any is stored
    const float* w1 = a.w1 + static_cast<size_t>(h) * HID * D2;
    constexpr int WL = HID * D2 / 4 / kScore64Threads;          // float4 loads per thread
    static_assert(WL >= 1 && WL * kScore64Threads == HID * D2 / 4, "whole loads per thread");
    float4 wv[WL];
#pragma unroll
    for (int x = 0; x < WL; ++x) {
      const int e = tid + x * kScore64Threads;
      wv[x] = __ldg(reinterpret_cast<const float4*>(w1 + static_cast<size_t>(e % HID) * D2) + e / HID);
    }
#pragma unroll
    for (int x = 0; x < WL; ++x) {
      const int e = tid + x * kScore64Threads;
      float* dst = Wt + (4 * (e / HID)) * WP + e % HID;
      dst[0] = wv[x].x;
      dst[WP] = wv[x].y;
      dst[2 * WP] = wv[x].z;
      dst[3 * WP] = wv[x].w;
    }
  }
  const int gr = lane >> 2, gc = lane & 3;                      // fragment row / column within a tile
  const int tg = warp & 3, hh = warp >> 2;                      // token group, hidden part
  const int j0 = hh * (HID / HS);
  // this lane's hidden units in the accumulators: j0 + 8 c + 2 gc + {0, 1}, c < NT
  double b1v[NT][2], w2v[NT][2];
#pragma unroll
  for (int c = 0; c < NT; ++c)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      b1v[c][e] = static_cast<double>(a.b1[static_cast<size_t>(h) * HID + j0 + 8 * c + 2 * gc + e]);
      w2v[c][e] = static_cast<double>(a.w2[static_cast<size_t>(h) * HID + j0 + 8 * c + 2 * gc + e]);
    }
  const double b2 = static_cast<double>(a.b2[h]);

  for (int tile = tile0; tile < tile0 + tpb && tile * TT < n_new; ++tile) {
    const int tok0 = tile * TT;
    __syncthreads();   // W1 written (first tile) / previous tile's reads done
    // the tile's rows, up to 8 16-byte loads in flight per thread before any is stored
    constexpr int XL = TT * UPT / kScore64Threads < 8 ? TT * UPT / kScore64Threads : 8;   // loads per batch
    static_assert(XL >= 1 && (TT * UPT) % (XL * kScore64Threads) == 0, "whole batches of loads");
#pragma unroll 1
    for (int e0 = 0; e0 < TT * UPT; e0 += XL * kScore64Threads) {
      uint4 raw[XL];
#pragma unroll
      for (int x = 0; x < XL; ++x) {
        const int e = e0 + tid + x * kScore64Threads;
        const int tt = e / UPT, c = e % UPT;
        raw[x] = make_uint4(0u, 0u, 0u, 0u);
        if (tok0 + tt < n_new) {
          const uint8_t* vs;
          const uint8_t* ks = token_row<T>(a, cg, u, cg.e0 + tok0 + tt, k, v, n, vs);
          const int i0 = c * EPU;
          raw[x] = *reinterpret_cast<const uint4*>((i0 < D2 / 2) ? ks + i0 * sizeof(T) : vs + (i0 - D2 / 2) * sizeof(T));
        }
      }
#pragma unroll
      for (int x = 0; x < XL; ++x) {
        const int e = e0 + tid + x * kScore64Threads;
        const int tt = e / UPT, c = e % UPT;
        const T* xe = reinterpret_cast<const T*>(&raw[x]);
#pragma unroll
        for (int q = 0; q < EPU; ++q) Xs[tt * XP + c * EPU + q] = Elem<T>::to_f32(xe[q]);
      }
    }
    __syncthreads();
    double acc[4][NT][2];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int c = 0; c < NT; ++c) acc[m][c][0] = acc[m][c][1] = 0.0;
    const float* xa = Xs + (32 * tg + gr) * XP + gc;              // A: row gr of tile m at + 8 m XP, inputs i0 + gc
    const float* wb = Wt + gc * WP + j0 + gr;                     // B: input i0 + gc, hidden j0 + 8 c + gr
#pragma unroll 2
    for (int i0 = 0; i0 < D2; i0 += 4) {
      double af[4], bf[NT];
#pragma unroll
      for (int m = 0; m < 4; ++m) af[m] = static_cast<double>(xa[8 * m * XP + i0]);
#pragma unroll
      for (int c = 0; c < NT; ++c) bf[c] = static_cast<double>(wb[i0 * WP + 8 * c]);
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int c = 0; c < NT; ++c) dmma_8x8x4(acc[m][c], af[m], bf[c]);
    }
    // w2 . relu(W1 x + b1) over this warp's hidden part: this lane holds
    // tokens 32 tg + 8 m + gr, 2 NT hidden units each
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      double part = 0.0;
#pragma unroll
      for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int e = 0; e < 2; ++e) part = fma(w2v[c][e], fmax(acc[m][c][e] + b1v[c][e], 0.0), part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (gc == 0) pp[hh * TT + 32 * tg + 8 * m + gr] = part;
    }
    __syncthreads();
    // the parts in a fixed order, + b2, one token per thread
    if (tid < TT && tok0 + tid < n_new) {
      double sum = pp[tid];
#pragma unroll
      for (int q = 1; q < HS; ++q) sum += pp[q * TT + tid];
      out[static_cast<size_t>(u) * cap + tok0 + tid] =
          ranking_priority(a, u, cg.e0 + tok0 + tid + a.W + a.D, static_cast<float>(sum + b2));
    }
  }
}

// score64_kernel for bf16 inputs, with each tile's rows copied while the
// tile before is computed.  The rows land by cp.async as they are (bf16
// pairs in 32-bit words, two buffers of TT rows) and are widened to fp64 as
// the fragments are loaded, so no thread waits for a tile's loads or
// converts it in shared memory.  W1 is kept transposed with the two inputs
// of each pair side by side (one 8-byte load per fragment serves two MMAs);
// in pass p0 lane (gr, gc) holds inputs 2 (p0 + gc) and 2 (p0 + gc) + 1 of
// its A row and B column, and the two MMAs of the pass take the first and
// the second of them: the same products, summed over the same inputs, as
// score64_kernel.  Row pitches: XW = 4 (mod 32) words and WP2 = 4 (mod 16)
// pairs keep every fragment load conflict-free.
template <int D2, int HID>
struct Score64BGeom {
  static constexpr int TT = 128;
  static constexpr int XW = D2 / 2 + 4;                       // 32-bit words per token row (16-byte multiple)
  static constexpr int WP2 = HID + 4;                         // float pairs per pair row of W1^T
  static constexpr size_t XBUF = static_cast<size_t>(TT) * XW * 4;
  static constexpr size_t W_OFF = 2 * XBUF;
  static constexpr size_t PP_OFF = W_OFF + static_cast<size_t>(D2 / 2) * WP2 * 8;
  static constexpr size_t SMEM = PP_OFF + 2 * static_cast<size_t>(kScore64Parts) * TT * 8;
  static_assert((XW * 4) % 16 == 0 && XW % 32 == 4 && WP2 % 16 == 4, "row pitches");
};

__device__ __forceinline__ void score_cp16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

template <int D2, int HID>
__global__ void __launch_bounds__(kScore64Threads, 1) score64_bf16_kernel(LayerArgs a, ChunkGeom cg,
                                                                          const __nv_bfloat16* __restrict__ k,
                                                                          const __nv_bfloat16* __restrict__ v,
                                                                          int n, float* __restrict__ out, int cap,
                                                                          int tpb) {
  using SG = Score64BGeom<D2, HID>;
  using T = __nv_bfloat16;
  constexpr int TT = SG::TT, XW = SG::XW, WP2 = SG::WP2;
  constexpr int HS = kScore64Parts;
  constexpr int NT = HID / (8 * HS);                            // column tiles of this warp's hidden part
  static_assert(NT >= 1 && HID % (8 * HS) == 0, "whole column tiles per part");
  constexpr int UPT = D2 / 8;                                   // 16-byte chunks per token row
  constexpr int CPT = TT * UPT / kScore64Threads;               // chunks per thread per tile
  static_assert(CPT >= 1 && CPT * kScore64Threads == TT * UPT, "whole chunks per thread");
  extern __shared__ __align__(16) uint8_t smb[];
  const uint32_t* Xw = reinterpret_cast<const uint32_t*>(smb);  // [buf][TT][XW]: bf16 pairs of x_t
  float2* Wt2 = reinterpret_cast<float2*>(smb + SG::W_OFF);     // [D2 / 2][WP2]: (W1[j][2p], W1[j][2p + 1])
  double* pp = reinterpret_cast<double*>(smb + SG::PP_OFF);     // [tile % 2][part][TT] partial sums
  const int u = blockIdx.y;
  const int h = u % a.Hkv;
  const int n_new = cg.e1 - cg.e0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile0 = blockIdx.x * tpb;
  const int ntile = min(tpb, (n_new + TT - 1) / TT - tile0);
  if (ntile <= 0) return;
  const uint32_t xs0 = smem_u32(smb);

  // a tile's rows into buffer b: thread -> chunks tid + x * threads (chunk c
  // of token tt = inputs 8 c .. 8 c + 7, from k for the first half of the
  // row, v for the second); tokens past the chunk's end are zero-filled
  auto issue = [&](int tile, int b) {
    const int tok0 = tile * TT;
#pragma unroll
    for (int x = 0; x < CPT; ++x) {
      const int e = tid + x * kScore64Threads;
      const int tt = e / UPT, c = e % UPT;
      const void* src = k;
      int bytes = 0;
      if (tok0 + tt < n_new) {
        const uint8_t* vs;
        const uint8_t* ks = token_row<T>(a, cg, u, cg.e0 + tok0 + tt, k, v, n, vs);
        const int i0 = c * 8;
        src = (i0 < D2 / 2) ? ks + i0 * sizeof(T) : vs + (i0 - D2 / 2) * sizeof(T);
        bytes = 16;
      }
      score_cp16(xs0 + static_cast<uint32_t>(b * SG::XBUF + (static_cast<size_t>(tt) * XW + c * 4) * 4), src, bytes);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(tile0, 0);

  {
    // W1 [HID][D2] -> Wt2 while the first tile is in flight: thread -> hidden
    // j = e % HID, inputs 4 q .. 4 q + 3 with q = e / HID (pairs 2 q, 2 q + 1)
    const float* w1 = a.w1 + static_cast<size_t>(h) * HID * D2;
    constexpr int WL = HID * D2 / 4 / kScore64Threads;          // float4 loads per thread
    static_assert(WL >= 1 && WL * kScore64Threads == HID * D2 / 4, "whole loads per thread");
    float4 wv[WL];
#pragma unroll
    for (int x = 0; x < WL; ++x) {
      const int e = tid + x * kScore64Threads;
      wv[x] = __ldg(reinterpret_cast<const float4*>(w1 + static_cast<size_t>(e % HID) * D2) + e / HID);
    }
#pragma unroll
    for (int x = 0; x < WL; ++x) {
      const int e = tid + x * kScore64Threads;
      float2* dst = Wt2 + (2 * (e / HID)) * WP2 + e % HID;
      dst[0] = make_float2(wv[x].x, wv[x].y);
      dst[WP2] = make_float2(wv[x].z, wv[x].w);
    }
  }
  const int gr = lane >> 2, gc = lane & 3;                      // fragment row / column within a tile
  const int tg = warp & 3, hh = warp >> 2;                      // token group, hidden part
  const int j0 = hh * (HID / HS);
  // this lane's hidden units in the accumulators: j0 + 8 c + 2 gc + {0, 1}, c < NT
  double b1v[NT][2], w2v[NT][2];
#pragma unroll
  for (int c = 0; c < NT; ++c)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      b1v[c][e] = static_cast<double>(a.b1[static_cast<size_t>(h) * HID + j0 + 8 * c + 2 * gc + e]);
      w2v[c][e] = static_cast<double>(a.w2[static_cast<size_t>(h) * HID + j0 + 8 * c + 2 * gc + e]);
    }
  const double b2 = static_cast<double>(a.b2[h]);

  // tile i's scores: the parts in a fixed order, + b2, one token per thread
  auto finish = [&](int i) {
    const int tok0 = (tile0 + i) * TT;
    const double* q = pp + (i & 1) * HS * TT;
    if (tid < TT && tok0 + tid < n_new) {
      double sum = q[tid];
#pragma unroll
      for (int x = 1; x < HS; ++x) sum += q[x * TT + tid];
      out[static_cast<size_t>(u) * cap + tok0 + tid] =
          ranking_priority(a, u, cg.e0 + tok0 + tid + a.W + a.D, static_cast<float>(sum + b2));
    }
  };
  for (int i = 0; i < ntile; ++i) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");       // this tile's rows
    // one barrier per tile: the rows (and W1) are visible, every thread is
    // done reading the other buffer (tile i - 1) and has written its parts
    // of tile i - 1, which are summed while tile i + 1's rows are copied
    __syncthreads();
    if (i > 0) finish(i - 1);
    if (i + 1 < ntile) issue(tile0 + i + 1, (i + 1) & 1);
    double acc[4][NT][2];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int c = 0; c < NT; ++c) acc[m][c][0] = acc[m][c][1] = 0.0;
    const uint32_t* xa = Xw + (i & 1) * TT * XW + (32 * tg + gr) * XW + gc;   // A: row gr of tile m at + 8 m XW
    const float2* wb = Wt2 + gc * WP2 + j0 + gr;                // B: pair row p0 + gc, hidden j0 + 8 c + gr
#pragma unroll 2
    for (int p0 = 0; p0 < D2 / 2; p0 += 4) {
      uint32_t aw[4];
      float2 bw[NT];
#pragma unroll
      for (int m = 0; m < 4; ++m) aw[m] = xa[8 * m * XW + p0];
#pragma unroll
      for (int c = 0; c < NT; ++c) bw[c] = wb[p0 * WP2 + 8 * c];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        double af[4], bf[NT];
#pragma unroll
        for (int m = 0; m < 4; ++m)
          af[m] = static_cast<double>(__uint_as_float(s == 0 ? aw[m] << 16 : aw[m] & 0xffff0000u));
#pragma unroll
        for (int c = 0; c < NT; ++c) bf[c] = static_cast<double>(s == 0 ? bw[c].x : bw[c].y);
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int c = 0; c < NT; ++c) dmma_8x8x4(acc[m][c], af[m], bf[c]);
      }
    }
    // w2 . relu(W1 x + b1) over this warp's hidden part: this lane holds
    // tokens 32 tg + 8 m + gr, 2 NT hidden units each
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      double part = 0.0;
#pragma unroll
      for (int c = 0; c < NT; ++c)
#pragma unroll
        for (int e = 0; e < 2; ++e) part = fma(w2v[c][e], fmax(acc[m][c][e] + b1v[c][e], 0.0), part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      if (gc == 0) pp[(i & 1) * HS * TT + hh * TT + 32 * tg + 8 * m + gr] = part;
    }
  }
  __syncthreads();
  finish(ntile - 1);
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// P1 with the stateless headwise linear scorer (page §E.2), s = w . [k; v] + b:
// one warp per token, the weight row in registers, fp64 dot product.
constexpr int kLinearThreads = 256;
constexpr int kLinearTokensPerWarp = 8;

template <typename T, int D2>
__global__ void __launch_bounds__(kLinearThreads) linear_score_kernel(LayerArgs a, ChunkGeom cg,
                                                                      const T* __restrict__ k,
                                                                      const T* __restrict__ v, int n,
                                                                      float* __restrict__ out, int cap) {
  const int u = blockIdx.y;
  const int h = u % a.Hkv;
  const int n_new = cg.e1 - cg.e0;
  const int warp = threadIdx.x >> 5;
  const int tok0 = (blockIdx.x * (kLinearThreads / 32) + warp) * kLinearTokensPerWarp;
  const float* w = head_w1(a, h);
  const float b = a.b2[h];
  for (int i = 0; i < kLinearTokensPerWarp; ++i) {
    const int r = tok0 + i;
    if (r >= n_new) break;
    const int t = cg.e0 + r;
    const uint8_t* vs;
    const uint8_t* ks = token_row<T>(a, cg, u, t, k, v, n, vs);
    const float s = linear_score_rows<T, D2>(reinterpret_cast<const T*>(ks), reinterpret_cast<const T*>(vs), w, b);
    if ((threadIdx.x & 31) == 0) out[static_cast<size_t>(u) * cap + r] = ranking_priority(a, u, t + a.W + a.D, s);
  }
}

// ---------------- P2: select + place ----------------
constexpr int kSelThreads = 1024;

// Exclusive block prefix sum of a 0/1 flag; returns the offset, sets *total.
__device__ __forceinline__ int block_scan_flag(int flag, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned ball = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(ball & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[warp] = __popc(ball);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int w = 0; w < nw; ++w) { const int c = warp_sums[w]; warp_sums[w] = run; run += c; }
    warp_sums[nw] = run;
  }
  __syncthreads();
  const int res = warp_sums[warp] + in_warp;
  *total = warp_sums[nw];
  __syncthreads();
  return res;
}

template <typename T>
__global__ void __launch_bounds__(kSelThreads) select_kernel(LayerArgs a, ChunkGeom cg, const T* __restrict__ k,
                                                             const T* __restrict__ v, int n,
                                                             const float* __restrict__ new_score, int cap,
                                                             int32_t* __restrict__ tgt_all) {
  __shared__ unsigned hist[256];
  __shared__ int warp_sums[kSelThreads / 32 + 1];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_need;
  __shared__ int s_list_tok[kSelThreads];
  __shared__ int s_list_slot[kSelThreads];

  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  const int K = a.K;
  const int base = topk_base(a.S, a.W, a.D);
  const int n_new = cg.e1 - cg.e0;
  const int c0 = cg.c0;
  int32_t* pos = a.pos + static_cast<size_t>(u) * a.NS;
  float* score = a.score + static_cast<size_t>(u) * a.NS;
  const float* ns = new_score + static_cast<size_t>(u) * cap;
  int32_t* tgt = tgt_all + static_cast<size_t>(u) * (K > 0 ? K : 1);
  uint8_t* kv = a.kv + static_cast<size_t>(u) * a.NS * a.row_bytes;

  if (tid == 0) {
    a.state[4 * u + 0] = cg.n1;
    a.state[4 * u + 1] = min(K, c0 + n_new);
  }
  if (n_new == 0 || K == 0) return;

  const int ncand = c0 + n_new;
  auto cand_key = [&](int i) -> unsigned long long {
    if (i < c0) return rank_key(score[base + i], pos[base + i]);
    return rank_key(ns[i - c0], cg.e0 + (i - c0));
  };

  unsigned long long thr = 0ull;   // admit keys >= thr
  if (ncand > K) {
    if (tid == 0) { s_prefix = 0ull; s_need = K; }
    unsigned long long mask = 0ull;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0u;
      __syncthreads();
      const unsigned long long prefix = s_prefix;
      for (int i = tid; i < ncand; i += blockDim.x) {
        const unsigned long long key = cand_key(i);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255ull], 1u);
      }
      __syncthreads();
      if (tid == 0) {
        int need = s_need;
        int cum = 0;
        int sel = 0;
        for (int dgt = 255; dgt >= 0; --dgt) {
          const int c = static_cast<int>(hist[dgt]);
          if (cum + c >= need) { sel = dgt; need -= cum; break; }
          cum += c;
        }
        s_need = need;
        s_prefix = prefix | (static_cast<unsigned long long>(sel) << shift);
      }
      mask |= 255ull << shift;
      __syncthreads();
    }
    thr = s_prefix;
  }

  // target slots: free or vacated long-range slots, ascending
  int n_tgt = 0;
  for (int i0 = 0; i0 < K; i0 += blockDim.x) {
    const int i = i0 + tid;
    int flag = 0;
    if (i < K) flag = (i >= c0) || (cand_key(i) < thr);
    int total;
    const int off = block_scan_flag(flag, warp_sums, &total);
    if (flag) tgt[n_tgt + off] = base + i;
    n_tgt += total;
  }
  __syncthreads();
  // admitted newcomers, ascending position -> tgt[rank]
  int n_adm = 0;
  for (int r0 = 0; r0 < n_new; r0 += blockDim.x) {
    const int r = r0 + tid;
    int flag = 0;
    if (r < n_new) flag = (ncand <= K) || (rank_key(ns[r], cg.e0 + r) >= thr);
    int total;
    const int off = block_scan_flag(flag, warp_sums, &total);
    if (flag) {
      s_list_tok[off] = cg.e0 + r;
      s_list_slot[off] = __ldcg(&tgt[n_adm + off]);
    }
    __syncthreads();
    // copy the rows: one warp per admitted token
    const int lane = tid & 31, warp = tid >> 5;
    for (int j = warp; j < total; j += blockDim.x / 32) {
      const int t = s_list_tok[j];
      const int slot = s_list_slot[j];
      const uint8_t* vs;
      const uint8_t* ks = token_row<T>(a, cg, u, t, k, v, n, vs);
      uint8_t* dst = kv + static_cast<size_t>(slot) * a.row_bytes;
      const int half = a.d * sizeof(T);
      for (int b = lane * 16; b < half; b += 32 * 16) {
        *reinterpret_cast<uint4*>(dst + b) = *reinterpret_cast<const uint4*>(ks + b);
        *reinterpret_cast<uint4*>(dst + half + b) = *reinterpret_cast<const uint4*>(vs + b);
      }
      if (lane == 0) {
        pos[slot] = t;
        score[slot] = ns[t - cg.e0];
      }
    }
    n_adm += total;
    __syncthreads();
  }
  // When the candidates overflow K every target slot is refilled
  // (|targets| == |admitted| == K - survivors); while filling up, the
  // admitted newcomers take the first free slots.
  if ((a.flags & FLAG_DEBUG_CHECKS) && tid == 0) {
    const bool bad = (ncand > K) ? (n_adm != n_tgt || n_adm > K) : (n_adm != n_new || n_adm > n_tgt);
    if (bad) set_error(a.err, DEVERR_STATE_MISMATCH);
  }
}

// ---------------- P3: window -> staging moves ----------------
template <typename T>
__global__ void move_kernel(LayerArgs a, ChunkGeom cg) {
  const int u = blockIdx.x;
  // window tokens before the chunk: [max(S, n0-W), n0); those in [n1-W-D, n1-W) now sit in staging
  const int lo = max(max(a.S, cg.n0 - a.W), cg.n1 - a.W - a.D);
  const int hi = min(cg.n0, cg.n1 - a.W);
  uint8_t* kv = a.kv + static_cast<size_t>(u) * a.NS * a.row_bytes;
  int32_t* pos = a.pos + static_cast<size_t>(u) * a.NS;
  float* score = a.score + static_cast<size_t>(u) * a.NS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = lo + warp; t < hi; t += blockDim.x / 32) {
    const int src = window_slot(t, a.S, a.W), dst = staging_slot(t, a.S, a.W, a.D);
    for (int b = lane * 16; b < a.row_bytes; b += 32 * 16)
      *reinterpret_cast<uint4*>(kv + static_cast<size_t>(dst) * a.row_bytes + b) =
          *reinterpret_cast<const uint4*>(kv + static_cast<size_t>(src) * a.row_bytes + b);
    if (lane == 0) { pos[dst] = t; score[dst] = score[src]; }
  }
}

// ---------------- P4: chunk tokens -> sink / window / staging ----------------
template <typename T>
__global__ void write_kernel(LayerArgs a, ChunkGeom cg, const T* __restrict__ k, const T* __restrict__ v, int n,
                             const float* __restrict__ ext) {
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = cg.n0 + blockIdx.x * (blockDim.x / 32) + warp;
  if (t >= cg.n1) return;
  int slot;
  if (t < a.S) slot = t;
  else if (t >= cg.n1 - a.W) slot = window_slot(t, a.S, a.W);
  else if (a.D > 0 && t >= cg.n1 - a.W - a.D) slot = staging_slot(t, a.S, a.W, a.D);
  else return;  // already eligible: handled by the select step
  uint8_t* dst = a.kv + (static_cast<size_t>(u) * a.NS + slot) * a.row_bytes;
  const size_t off = (static_cast<size_t>(u) * n + (t - cg.n0)) * a.d;
  const uint8_t* ks = reinterpret_cast<const uint8_t*>(k + off);
  const uint8_t* vs = reinterpret_cast<const uint8_t*>(v + off);
  const int half = a.d * sizeof(T);
  for (int b = lane * 16; b < half; b += 32 * 16) {
    *reinterpret_cast<uint4*>(dst + b) = *reinterpret_cast<const uint4*>(ks + b);
    *reinterpret_cast<uint4*>(dst + half + b) = *reinterpret_cast<const uint4*>(vs + b);
  }
  if (lane == 0) {
    a.pos[static_cast<size_t>(u) * a.NS + slot] = t;
    a.score[static_cast<size_t>(u) * a.NS + slot] =
        (a.flags & FLAG_EXTERNAL_SCORES) ? ext[static_cast<size_t>(u) * n + (t - cg.n0)] : 0.f;
  }
}

template <typename T, int D2, int HID>
int launch_score64(const LayerArgs& a, const ChunkGeom& cg, const T* k, const T* v, int n, float* out, int cap,
                   int n_new, cudaStream_t st) {
  // the shared-memory attribute is set on every call: it belongs to the current device
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return -1;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    using SG = Score64BGeom<D2, HID>;
    if (cudaFuncSetAttribute(score64_bf16_kernel<D2, HID>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(SG::SMEM)) != cudaSuccess)
      return -1;
    const int tiles = (n_new + SG::TT - 1) / SG::TT;
    const int tpb = score64_tiles_per_block(tiles, a.units, nsm);
    dim3 grid((tiles + tpb - 1) / tpb, a.units);
    score64_bf16_kernel<D2, HID><<<grid, kScore64Threads, SG::SMEM, st>>>(a, cg, k, v, n, out, cap, tpb);
  } else {
    using SG = Score64Geom<D2, HID>;
    if (cudaFuncSetAttribute(score64_kernel<T, D2, HID>, cudaFuncAttributeMaxDynamicSharedMemorySize, SG::SMEM) !=
        cudaSuccess)
      return -1;
    const int tiles = (n_new + SG::TT - 1) / SG::TT;
    const int tpb = score64_tiles_per_block(tiles, a.units, nsm);
    dim3 grid((tiles + tpb - 1) / tpb, a.units);
    score64_kernel<T, D2, HID><<<grid, kScore64Threads, SG::SMEM, st>>>(a, cg, k, v, n, out, cap, tpb);
  }
  return 0;
}

// P1 for the tokens [cg.e0, cg.e1): ranking priority of each into out[u * cap + (t - cg.e0)].
template <typename T>
int launch_scores_t(const LayerArgs& a, const ChunkGeom& cg, const T* k, const T* v, int n, const float* ext,
                    float* out, int cap, cudaStream_t st) {
  const int n_new = cg.e1 - cg.e0;
  const bool use64 = !(a.flags & FLAG_EXTERNAL_SCORES) && (a.hidden == 32 || a.hidden == 64) &&
                     (a.d == 64 || a.d == 128);
  if (n_new > 0 && use64) {
    int r = 0;
    if (a.d == 128 && a.hidden == 64) r = launch_score64<T, 256, 64>(a, cg, k, v, n, out, cap, n_new, st);
    else if (a.d == 128) r = launch_score64<T, 256, 32>(a, cg, k, v, n, out, cap, n_new, st);
    else if (a.hidden == 64) r = launch_score64<T, 128, 64>(a, cg, k, v, n, out, cap, n_new, st);
    else r = launch_score64<T, 128, 32>(a, cg, k, v, n, out, cap, n_new, st);
    if (r != 0) return r;
  } else if (n_new > 0 && a.hidden == 0 && !(a.flags & FLAG_EXTERNAL_SCORES)) {
    constexpr int per_block = (kLinearThreads / 32) * kLinearTokensPerWarp;
    dim3 grid((n_new + per_block - 1) / per_block, a.units);
    if (a.d == 128)
      linear_score_kernel<T, 256><<<grid, kLinearThreads, 0, st>>>(a, cg, k, v, n, out, cap);
    else
      linear_score_kernel<T, 128><<<grid, kLinearThreads, 0, st>>>(a, cg, k, v, n, out, cap);
  } else if (n_new > 0) {
    const int HQ = a.hidden / 4;
    const int TT = 4 * (kScoreThreads / HQ);
    const size_t smem = (a.flags & FLAG_EXTERNAL_SCORES) ? 0
                        : (static_cast<size_t>(2 * a.d) * a.hidden + static_cast<size_t>(TT) * 2 * a.d) * sizeof(float);
    if (smem > 48 * 1024 && cudaFuncSetAttribute(score_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(smem)) != cudaSuccess)
      return -1;
    dim3 grid((n_new + TT - 1) / TT, a.units);
    score_kernel<T><<<grid, kScoreThreads, smem, st>>>(a, cg, k, v, n, ext, out, cap);
  }
  return 0;
}

template <typename T>
int launch_prefill_t(const LayerArgs& a, const PrefillScratch& ps, const T* k, const T* v, int n, int n0, int c0,
                     const float* ext, cudaStream_t st) {
  ChunkGeom cg;
  cg.n0 = n0;
  cg.n1 = n0 + n;
  cg.e0 = max(a.S, n0 - a.W - a.D);
  cg.e1 = max(a.S, cg.n1 - a.W - a.D);
  cg.c0 = c0;
  const int n_new = cg.e1 - cg.e0;
  if (n_new > ps.cap) return -2;
  const int r = a.mlstm ? launch_mlstm_prefill(a, sizeof(T) == 4 ? 0 : 1, k, v, n, n0, cg.e0, ps.new_score, ps.cap, st)
                        : launch_scores_t<T>(a, cg, k, v, n, ext, ps.new_score, ps.cap, st);
  if (r != 0) return r;
  select_kernel<T><<<a.units, kSelThreads, 0, st>>>(a, cg, k, v, n, ps.new_score, ps.cap, ps.tgt);
  if (a.D > 0) move_kernel<T><<<a.units, 256, 0, st>>>(a, cg);
  if (n > 0) {
    dim3 grid((n + 7) / 8, a.units);
    write_kernel<T><<<grid, 256, 0, st>>>(a, cg, k, v, n, ext);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_prompt_scores(const LayerArgs& a, int dtype, const void* k, const void* v, int n, const float* ext,
                         float* out, int cap, cudaStream_t st) {
  ChunkGeom cg;
  cg.n0 = 0;
  cg.n1 = n;
  cg.e0 = a.S;
  cg.e1 = max(a.S, n - a.W - a.D);
  cg.c0 = 0;
  if (cg.e1 - cg.e0 > cap) return -2;
  int r;
  if (dtype == 0)
    r = launch_scores_t<float>(a, cg, static_cast<const float*>(k), static_cast<const float*>(v), n, ext, out, cap, st);
  else
    r = launch_scores_t<__nv_bfloat16>(a, cg, static_cast<const __nv_bfloat16*>(k),
                                       static_cast<const __nv_bfloat16*>(v), n, ext, out, cap, st);
  if (r != 0) return r;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_prompt_write(const LayerArgs& a, int dtype, const void* k, const void* v, int n, const float* ext,
                        cudaStream_t st) {
  ChunkGeom cg;
  cg.n0 = 0;
  cg.n1 = n;
  cg.e0 = a.S;
  cg.e1 = max(a.S, n - a.W - a.D);
  cg.c0 = 0;
  if (n <= 0) return 0;
  dim3 grid((n + 7) / 8, a.units);
  if (dtype == 0)
    write_kernel<float><<<grid, 256, 0, st>>>(a, cg, static_cast<const float*>(k), static_cast<const float*>(v), n, ext);
  else
    write_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a, cg, static_cast<const __nv_bfloat16*>(k),
                                                      static_cast<const __nv_bfloat16*>(v), n, ext);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_prefill(const LayerArgs& a, int dtype, const PrefillScratch& ps, const void* k, const void* v,
                   int n_tokens, int n_seen_before, int n_topk_before, const float* ext_scores, cudaStream_t st) {
  if (dtype == 0)
    return launch_prefill_t<float>(a, ps, static_cast<const float*>(k), static_cast<const float*>(v), n_tokens,
                                   n_seen_before, n_topk_before, ext_scores, st);
  return launch_prefill_t<__nv_bfloat16>(a, ps, static_cast<const __nv_bfloat16*>(k),
                                         static_cast<const __nv_bfloat16*>(v), n_tokens, n_seen_before,
                                         n_topk_before, ext_scores, st);
}

}  // namespace kvpop
