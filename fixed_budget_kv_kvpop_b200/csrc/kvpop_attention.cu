// Split-K flash-decode over the slot-addressed KVpop cache.
//
// Decoding attends directly over the retained cache entries (KVpop page §C.1
// Mask Definition): for each (batch row, KV head) unit, the G query heads of
// the group attend over every occupied slot (sinks, window, staging ring,
// long-range top-k).  Scale 1/sqrt(d), fp32 accumulation.
//
// Design (sm_100a, HBM-bound GEMV; no tensor cores):
//  * Persistent grid, one CTA per SM: 8 consumer warps + 1 producer warp.
//  * The tiles of all units (16 slots = 16 contiguous rows of [k | v]) form one
//    flat sequence that is cut into equal contiguous ranges, one per consumer
//    warp ("stream-K"), so every warp streams the same number of bytes.
//  * The producer's elected lane moves each tile with one cp.async.bulk
//    (no multicast) into the owning warp's 3-deep shared-memory ring;
//    completion is tracked by mbarrier transaction bytes.
//  * A consumer warp is 4 groups of 8 lanes.  A group takes 4 slots of a tile;
//    each lane owns 16 dims (two 16-byte chunks per row), keeps its slice of the
//    G queries in registers, and the 8 partial dot products are all-reduced
//    with 3 butterfly shuffles.  Each group keeps its own online-softmax state
//    (running max m, sum l, fp32 accumulators), so no cross-group traffic
//    happens in the main loop.
//  * When a warp's range leaves a unit it folds its 4 groups together and
//    writes one partial (m, l, acc) per head.  The last warp to finish a unit
//    (atomic ticket, no waiting) merges the partials with a log-sum-exp
//    combine and writes the output.  Units covered by a single warp are
//    written directly.
#include "kvpop_internal.cuh"

namespace kvpop {

namespace {

constexpr int NCW = kConsumerWarps;
constexpr int NSTG = kStagesPerWarp;
constexpr int TS = kTileSlots;
constexpr int kThreads = (NCW + 1) * 32;
constexpr float kNegInf = -__builtin_huge_valf();

template <typename T, int DH>
struct Geo {
  static constexpr int ESZ = sizeof(T);
  static constexpr int ROW = 2 * DH * ESZ;          // bytes per slot row [k | v]
  static constexpr int NCHK = DH * ESZ / 16;        // 16-byte chunks per k row
  static constexpr int CPL = NCHK / 8;              // chunks per lane
  static constexpr int EPC = 16 / ESZ;              // elements per chunk
  static constexpr int DPL = CPL * EPC;             // dims per lane
  static constexpr int STAGE_BYTES = TS * ROW;
  static_assert(NCHK % 8 == 0 && CPL >= 1, "row must be a multiple of 128 bytes");
};

struct ValidGeom {
  int p, S, W, D, nse;
  bool full;
  __device__ __forceinline__ bool slot_ok(int i) const {
    if (i >= nse) return false;
    if (full) return true;
    if (i < S) return i <= p;
    if (i < S + W) {
      if (p < S) return false;
      int idx = i - S;
      int t = p - (((p - idx) % W) + W) % W;
      return t >= S;
    }
    if (i < S + W + D) {
      int q0 = p - W;
      if (q0 < S) return false;
      int idx = i - S - W;
      int t = q0 - (((q0 - idx) % D) + D) % D;
      return t >= S;
    }
    return true;  // long-range slots below nse are occupied
  }
};

template <typename T, int DH, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_attention_kernel(const LayerArgs a, const DecodeScratch sc, const T* __restrict__ q, T* __restrict__ out) {
  using GE = Geo<T, DH>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + NCW * NSTG * GE::STAGE_BYTES);
  uint64_t* empty_bar = full_bar + NCW * NSTG;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- geometry of this step (identical in every thread) ----
  const int n_seen = a.state[0];
  const int ntk = a.state[1];
  ValidGeom vg;
  vg.p = n_seen - 1; vg.S = a.S; vg.W = a.W; vg.D = a.D;
  vg.nse = a.S + a.W + a.D + ntk;
  vg.full = n_seen >= a.S + a.W + a.D;
  const int64_t tpu = (vg.nse + TS - 1) / TS;
  const int64_t total = static_cast<int64_t>(a.units) * tpu;
  const int64_t nw = decode_active_warps(total, tpu, static_cast<int64_t>(gridDim.x) * NCW);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NCW * NSTG; ++i) { mbar_init(&full_bar[i], 1); mbar_init(&empty_bar[i], 1); }
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == NCW) {
    // ---------------- producer ----------------
    if (lane != 0) return;
    int64_t lo[NCW], cnt[NCW];
    int64_t maxc = 0;
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      const int64_t gw = static_cast<int64_t>(blockIdx.x) * NCW + w;
      if (gw < nw) { lo[w] = seg_lo(gw, total, nw); cnt[w] = seg_lo(gw + 1, total, nw) - lo[w]; }
      else { lo[w] = 0; cnt[w] = 0; }
      maxc = cnt[w] > maxc ? cnt[w] : maxc;
    }
    for (int64_t i = 0; i < maxc; ++i) {
      const int stage = static_cast<int>(i % NSTG);
      const uint32_t round = static_cast<uint32_t>(i / NSTG);
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        if (i >= cnt[w]) continue;
        if (round > 0 && !mbar_wait(&empty_bar[w * NSTG + stage], (round - 1) & 1)) {
          set_error(a.err, DEVERR_TIMEOUT);
          return;
        }
        const int64_t t = lo[w] + i;
        const int64_t unit = t / tpu;
        const int s0 = static_cast<int>(t - unit * tpu) * TS;
        const int nslots = min(TS, vg.nse - s0);
        const uint32_t bytes = static_cast<uint32_t>(nslots) * GE::ROW;
        uint8_t* dst = smem + (w * NSTG + stage) * GE::STAGE_BYTES;
        const uint8_t* src = a.kv + (unit * a.NS + s0) * static_cast<int64_t>(GE::ROW);
        mbar_arrive_expect_tx(&full_bar[w * NSTG + stage], bytes);
        bulk_g2s(dst, src, bytes, &full_bar[w * NSTG + stage]);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * NCW + warp;
  if (gw >= nw) return;
  const int64_t lo = seg_lo(gw, total, nw);
  const int64_t hi = seg_lo(gw + 1, total, nw);
  const int grp = lane >> 3;   // 0..3
  const int sub = lane & 7;    // 0..7
  const float qscale = 1.4426950408889634f * rsqrtf(static_cast<float>(DH));

  float qr[G][GE::DPL];
  float acc[G][GE::DPL];
  float m[G], l[G];
  int64_t cur = -1;

  auto load_q = [&](int64_t unit) {
    const T* qu = q + unit * (G * DH);
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int r = 0; r < GE::CPL; ++r) {
        const uint4 raw = *reinterpret_cast<const uint4*>(qu + g * DH + (sub + 8 * r) * GE::EPC);
        float f[GE::EPC];
        unpack16(raw, f, T());
#pragma unroll
        for (int e = 0; e < GE::EPC; ++e) qr[g][r * GE::EPC + e] = f[e] * qscale;
      }
      m[g] = kNegInf; l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < GE::DPL; ++e) acc[g][e] = 0.f;
    }
  };

  auto finalize = [&](int64_t unit) {
    // fold the 4 groups of the warp
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
        const float lo_ = __shfl_xor_sync(0xffffffffu, l[g], off);
        const float M = fmaxf(m[g], mo);
        const float c1 = (m[g] == kNegInf) ? 0.f : exp2f(m[g] - M);
        const float c2 = (mo == kNegInf) ? 0.f : exp2f(mo - M);
        l[g] = l[g] * c1 + lo_ * c2;
#pragma unroll
        for (int e = 0; e < GE::DPL; ++e) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], off);
          acc[g][e] = acc[g][e] * c1 + ao * c2;
        }
        m[g] = M;
      }
    }
    const int64_t first = warp_of_tile(unit * tpu, total, nw);
    const int64_t last = warp_of_tile(unit * tpu + tpu - 1, total, nw);
    const int nseg = static_cast<int>(last - first + 1);
    T* ou = out + unit * (G * DH);
    if (nseg == 1) {
      if (grp == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float inv = l[g] > 0.f ? 1.f / l[g] : 0.f;
#pragma unroll
          for (int r = 0; r < GE::CPL; ++r)
#pragma unroll
            for (int e = 0; e < GE::EPC; ++e)
              ou[g * DH + (sub + 8 * r) * GE::EPC + e] = Elem<T>::from_f32(acc[g][r * GE::EPC + e] * inv);
        }
      }
      return;
    }
    const int seg = static_cast<int>(gw - first);
    if (seg >= kMaxSeg || nseg > kMaxSeg) {  // cannot happen: decode_active_warps bounds nseg
      if (lane == 0) set_error(a.err, DEVERR_BAD_INDEX);
      return;
    }
    float* pa = sc.part_acc + (unit * kMaxSeg + seg) * (G * DH);
    float* pm = sc.part_ml + (unit * kMaxSeg + seg) * (G * 2);
    if (grp == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int r = 0; r < GE::CPL; ++r)
#pragma unroll
          for (int e = 0; e < GE::EPC; ++e)
            pa[g * DH + (sub + 8 * r) * GE::EPC + e] = acc[g][r * GE::EPC + e];
      if (sub == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) { pm[2 * g] = m[g]; pm[2 * g + 1] = l[g]; }
      }
    }
    __threadfence();
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = atomicAdd(&sc.ticket[unit], 1);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != nseg - 1) return;
    // last arrival: merge all partials of this unit
    __threadfence();
    const float* pab = sc.part_acc + unit * kMaxSeg * (G * DH);
    const float* pmb = sc.part_ml + unit * kMaxSeg * (G * 2);
    for (int g = 0; g < G; ++g) {
      float M = kNegInf;
      for (int s = 0; s < nseg; ++s) M = fmaxf(M, __ldcg(pmb + s * G * 2 + 2 * g));
      float L = 0.f;
      for (int s = 0; s < nseg; ++s) {
        const float ms = __ldcg(pmb + s * G * 2 + 2 * g);
        if (ms != kNegInf) L += __ldcg(pmb + s * G * 2 + 2 * g + 1) * exp2f(ms - M);
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      for (int dd = lane; dd < DH; dd += 32) {
        float o = 0.f;
        for (int s = 0; s < nseg; ++s) {
          const float ms = __ldcg(pmb + s * G * 2 + 2 * g);
          if (ms != kNegInf) o += __ldcg(pab + s * G * DH + g * DH + dd) * exp2f(ms - M);
        }
        ou[g * DH + dd] = Elem<T>::from_f32(o * inv);
      }
    }
    if (lane == 0) sc.ticket[unit] = 0;
  };

  for (int64_t t = lo; t < hi; ++t) {
    const int64_t i = t - lo;
    const int stage = static_cast<int>(i % NSTG);
    const int64_t unit = t / tpu;
    if (unit != cur) {
      if (cur >= 0) finalize(cur);
      cur = unit;
      load_q(unit);
    }
    if (!mbar_wait(&full_bar[warp * NSTG + stage], static_cast<uint32_t>(i / NSTG) & 1)) {
      if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
      return;
    }
    const uint8_t* tile = smem + (warp * NSTG + stage) * GE::STAGE_BYTES;
    const int s0 = static_cast<int>(t - unit * tpu) * TS;

    float s[4][G];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      const uint4* krow = reinterpret_cast<const uint4*>(tile + (grp + 4 * tt) * GE::ROW);
#pragma unroll
      for (int g = 0; g < G; ++g) s[tt][g] = 0.f;
#pragma unroll
      for (int r = 0; r < GE::CPL; ++r) {
        const uint4 raw = krow[sub + 8 * r];
        float kf[GE::EPC];
        unpack16(raw, kf, T());
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < GE::EPC; ++e) s[tt][g] = fmaf(qr[g][r * GE::EPC + e], kf[e], s[tt][g]);
      }
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1)
#pragma unroll
      for (int tt = 0; tt < 4; ++tt)
#pragma unroll
        for (int g = 0; g < G; ++g) s[tt][g] += __shfl_xor_sync(0xffffffffu, s[tt][g], off);

    bool ok[4];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      ok[tt] = vg.slot_ok(s0 + grp + 4 * tt);
      if (!ok[tt]) {
#pragma unroll
        for (int g = 0; g < G; ++g) s[tt][g] = kNegInf;
      }
    }
    float pr[4][G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mt = fmaxf(fmaxf(s[0][g], s[1][g]), fmaxf(s[2][g], s[3][g]));
      const float mn = fmaxf(m[g], mt);
      if (mn == kNegInf) {
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) pr[tt][g] = 0.f;
        continue;
      }
      const float alpha = exp2f(m[g] - mn);   // m = -inf -> 0
      float sum = 0.f;
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) { pr[tt][g] = exp2f(s[tt][g] - mn); sum += pr[tt][g]; }
      l[g] = l[g] * alpha + sum;
      m[g] = mn;
#pragma unroll
      for (int e = 0; e < GE::DPL; ++e) acc[g][e] *= alpha;
    }
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      if (!ok[tt]) continue;
      const uint4* vrow = reinterpret_cast<const uint4*>(tile + (grp + 4 * tt) * GE::ROW + DH * GE::ESZ);
#pragma unroll
      for (int r = 0; r < GE::CPL; ++r) {
        const uint4 raw = vrow[sub + 8 * r];
        float vf[GE::EPC];
        unpack16(raw, vf, T());
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < GE::EPC; ++e)
            acc[g][r * GE::EPC + e] = fmaf(pr[tt][g], vf[e], acc[g][r * GE::EPC + e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[warp * NSTG + stage]);
  }
  if (cur >= 0) finalize(cur);
}

template <typename T, int DH, int G>
int launch_t(const LayerArgs& a, const DecodeScratch& sc, const void* q, void* out, int num_sms, cudaStream_t st) {
  using GE = Geo<T, DH>;
  const size_t smem = static_cast<size_t>(NCW) * NSTG * GE::STAGE_BYTES + 2 * NCW * NSTG * sizeof(uint64_t);
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(decode_attention_kernel<T, DH, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return -1;
    attr_set = true;
  }
  const int64_t tpu_max = (a.NS + TS - 1) / TS;
  const int64_t total_max = static_cast<int64_t>(a.units) * tpu_max;
  int64_t grid = (total_max + NCW - 1) / NCW;
  if (grid > num_sms) grid = num_sms;
  if (grid < 1) grid = 1;
  decode_attention_kernel<T, DH, G><<<static_cast<int>(grid), kThreads, smem, st>>>(
      a, sc, static_cast<const T*>(q), static_cast<T*>(out));
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int attention_supported(int dtype, int d, int G) {
  if (dtype == 1 && d == 128) return G == 1 || G == 2 || G == 4;
  if (d == 64) return G == 1 || G == 2 || G == 4 || G == 8;
  return 0;
}

int launch_attention(const LayerArgs& a, int dtype, const DecodeScratch& sc, const void* q, void* out,
                     int num_sms, cudaStream_t st) {
#define KVPOP_DISPATCH(TT, DD, GG) \
  if (a.d == DD && a.G == GG) return launch_t<TT, DD, GG>(a, sc, q, out, num_sms, st);
  if (dtype == 1) {
    KVPOP_DISPATCH(__nv_bfloat16, 128, 4)
    KVPOP_DISPATCH(__nv_bfloat16, 128, 2)
    KVPOP_DISPATCH(__nv_bfloat16, 128, 1)
    KVPOP_DISPATCH(__nv_bfloat16, 64, 8)
    KVPOP_DISPATCH(__nv_bfloat16, 64, 4)
    KVPOP_DISPATCH(__nv_bfloat16, 64, 2)
    KVPOP_DISPATCH(__nv_bfloat16, 64, 1)
  } else {
    KVPOP_DISPATCH(float, 64, 8)
    KVPOP_DISPATCH(float, 64, 4)
    KVPOP_DISPATCH(float, 64, 2)
    KVPOP_DISPATCH(float, 64, 1)
  }
#undef KVPOP_DISPATCH
  return -2;
}

}  // namespace kvpop
