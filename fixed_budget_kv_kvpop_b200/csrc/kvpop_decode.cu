// KVpop decode step: fused cache update + split-K flash decode (sm_100a).
//
// Method: KVpop page §3 (fixed-budget pruning), §C.1 (mask definition:
// decoding attends directly over the retained cache entries: sinks, recent
// window, selected long-range tokens), §E.1-§E.2 (headwise MLP scorer on
// [k; v]), §E.4 / §I (a token is scored when it reaches the eviction
// boundary u = q - w; with delayed scoring D more steps later).
//
// One launch per layer and step does all of it.  The step that appends token
// N (position p = N) changes the attended set by exactly one token out and
// one in: the boundary token b = N - W - D either replaces the long-range
// minimum e (e leaves) or is dropped (b leaves), and the new token N enters;
// every other token only changes slot.  So the kernel
//   * attends over the cache as it stood after step N-1, masking the single
//     slot `evict` of this step's decision, and adds the new token's (k, v)
//     from the input as one extra term in the final merge;
//   * takes the NEXT step's eviction decision (score of token N+1-W-D, block
//     argmin of the long-range keys, with this step's replacement applied) in
//     a dedicated decider warp while the other warps stream the cache;
//   * lets the last warp to finish a unit merge the split-K partials, write
//     the output and commit this step's row moves (boundary token into its
//     long-range slot, window token into the staging ring, new token into its
//     window slot), after every reader of those rows has finished.
// MODE_ATTEND is the attention part alone over the cache as it stands.
//
// Streaming layout: the tiles of all units (16 slots, one 2*d*sizeof(T) row
// [k | v] per slot) form one sequence cut into equal contiguous ranges, one
// per consumer warp (stream-K).  Each consumer warp feeds its own shared-memory
// ring (NSTG stages of one tile): the layer's rows are one 2-D tensor map
// (inner dimension 2*d elements, outer units*NS rows) and a tile is 2*d*size/128
// TMA boxes of 16 rows x 128 bytes with the 128-byte swizzle, issued by that
// many lanes (cp.async.bulk.tensor, no multicast), completion counted on the
// stage's mbarrier.  The swizzle makes the row-per-lane QK reads and the
// chunk-per-lane PV reads of 16-byte vectors conflict-free.
// QK: lane (j, h) computes slot j's dot products over half h of the dims for
// all G heads, q broadcast from shared memory, packed fp32 FMA
// (fma.rn.f32x2); one shuffle joins the halves.  Softmax in the exp2 domain
// with lazy rescaling (the running max moves only when a tile exceeds it by
// 2^8).  PV: lanes own 16-byte chunks of the value row, slot groups split the
// tile, p broadcast from shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kvpop_internal.cuh"

namespace kvpop {

namespace {

constexpr int TS = 16;                               // slots per tile
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kLazy = 8.0f;                        // lazy rescale threshold (log2 units)
constexpr float kLog2e = 1.4426950408889634f;

// Launch shape of the decode kernel: consumer warps per CTA, shared-memory
// stages per consumer warp, decider warps per CTA.  bf16 consumers run both
// contractions on the tensor cores and need few warps to keep HBM busy;
// keeping fewer tiles in flight also keeps the memory latency that the
// deciders' dependent loads and the merges see short.  fp32 consumers (FMA
// pipes) are issue-bound and take more warps.
template <typename T, int G>
struct LaunchShape {
  static constexpr int NCW = sizeof(T) == 2 ? 6 : (G > 4 ? 8 : 10);
  static constexpr int NSTG = 2;
  static constexpr int NDW = sizeof(T) == 2 ? 4 : 2;
};
constexpr int kMaxDeciders = 8;   // decider warps per CTA at most (team slots in shared memory)
// Tiles per consumer warp prefetched into L2 before the wait for the previous kernel.
constexpr int kPrefetchTiles = 2;

// A tile is TS rows [k | v]; it lands in shared memory as NBLK boxes of
// TS rows x 128 bytes (box b holds bytes [128 b, 128 b + 128) of every row),
// swizzled by the tensor-map TMA: 16-byte chunk c of box row j sits at chunk
// c ^ (j & 7).  Column reads of 8 consecutive rows and row reads of 8
// consecutive chunks both hit 8 distinct bank groups.
template <typename T, int DH, int G>
struct Geo {
  static constexpr int ESZ = sizeof(T);
  static constexpr int ROW = 2 * DH * ESZ;      // bytes per slot row [k | v]
  static constexpr int NCHK = DH * ESZ / 16;    // 16-byte chunks per k (or v) row
  static constexpr int NBLK = ROW / 128;        // 128-byte boxes per row
  static constexpr int BOX = TS * 128;          // bytes per box in shared memory
  static constexpr int BOXELEMS = 128 / ESZ;    // elements per box row
  static constexpr int CH = NCHK / 2;           // chunks per QK half
  static constexpr int EPC = 16 / ESZ;          // elements per chunk
  static constexpr int LPS = NCHK;              // PV: lanes per slot
  static constexpr int SG = 32 / LPS;           // PV: slot groups
  static constexpr int SPG = TS / SG;           // PV: slots per group
  static constexpr int STAGE = TS * ROW;
  static constexpr int QHALF = CH * G * EPC * 4;     // bytes of one q half
  static constexpr int QBYTES = 2 * QHALF + 16;      // + pad between halves
  static constexpr int PSLOT = 2 * G * 4;            // p pairs (p, p) per slot
  static constexpr int PBYTES = TS * PSLOT + SG * 16;
  static_assert(NCHK == 8 || NCHK == 16, "k row must be 128 or 256 bytes");
  // byte offset of 16-byte chunk c (0 <= c < 2 NCHK; v row from NCHK) of slot j
  static __device__ __forceinline__ int off(int j, int c) {
    return (c >> 3) * BOX + j * 128 + (((c & 7) ^ (j & 7)) << 4);
  }
};

constexpr int kMergeCap = 512;   // per-CTA ring of units ready to merge

template <typename T, int DH, int G, int NCW, int NSTG>
struct Smem {
  using GE = Geo<T, DH, G>;
  static constexpr int QRB = (G * DH + 2 * DH) * GE::ESZ + 32;   // raw q | k_new | v_new | decision of one unit
  static constexpr int RINGS = 0;
  static constexpr int Q = RINGS + NCW * NSTG * GE::STAGE;
  static constexpr int P = Q + NCW * GE::QBYTES;
  static constexpr int QRAW = P + NCW * GE::PBYTES;
  static constexpr int MQ = QRAW + NCW * 2 * QRB;
  static constexpr int BAR = MQ + (kMergeCap + 4) * 4;
  static constexpr int TEAM = BAR + NCW * (NSTG + 2) * 8;             // the deciders' parts (decide_finish in teams)
  static constexpr int TOTAL = TEAM + kMaxDeciders * 24;
  static_assert(GE::STAGE % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
  static_assert(Q % 16 == 0 && P % 16 == 0 && QRAW % 16 == 0 && QRB % 16 == 0 && MQ % 16 == 0 &&
                    BAR % 8 == 0,
                "smem alignment");
  static_assert(TOTAL <= 232448, "shared memory per CTA exceeds 227 KB");
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Ticket increment with acquire-release semantics at GPU scope: the caller's
// (and, after __syncwarp, its warp's) earlier writes are visible to whoever
// observes the new count.
__device__ __forceinline__ int ticket_add(int32_t* t) {
  int prev;
  asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], 1;" : "=r"(prev) : "l"(t) : "memory");
  return prev;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Validity of a slot of the cache holding tokens 0..p (fill-up phases only).
struct ValidGeom {
  int p, S, W, D, nse;
  bool full;
  __device__ __forceinline__ bool slot_ok(int i) const {
    if (i >= nse) return false;
    if (full) return true;
    if (i < S) return i <= p;
    if (i < S + W) {
      if (p < S) return false;
      const int idx = i - S;
      const int t = p - (((p - idx) % W) + W) % W;
      return t >= S;
    }
    if (i < S + W + D) {
      const int q0 = p - W;
      if (q0 < S) return false;
      const int idx = i - S - W;
      const int t = q0 - (((q0 - idx) % D) + D) % D;
      return t >= S;
    }
    return true;  // long-range slots below nse are occupied
  }
};

// Eviction decision for the step that appends token N, taken by one warp.
// pending == nullptr: the cache as committed (holds tokens 0..N-1).
// pending != nullptr: the cache before the commit of the step appending token
// N-1 (described by *pending); token N-1 is then (kn, vn, ext_new).
// ntk = long-range slots in use once that step is committed.
template <typename T>
__device__ __noinline__ Decision decide_warp(const LayerArgs& a, int u, int N, int ntk, const Decision* pending,
                                const T* kn, const T* vn, float ext_new) {
  const int lane = threadIdx.x & 31;
  const int S = a.S, W = a.W, D = a.D, NS = a.NS;
  Decision r;
  r.p = N; r.bpos = -1; r.bslot = -1; r.tgt = -1; r.evict = -1; r.sb = 0.f; r.pad[0] = r.pad[1] = 0;
  const int b = N - W - D;
  if (b < S) return r;
  const T* kv = reinterpret_cast<const T*>(a.kv + static_cast<size_t>(u) * NS * a.row_bytes);
  const int32_t* pos = a.pos + static_cast<size_t>(u) * NS;
  const float* score = a.score + static_cast<size_t>(u) * NS;
  r.bpos = b;
  r.bslot = (D == 0) ? window_slot(b, S, W) : staging_slot(b, S, W, D);
  // where b's row is now
  const T* krow;
  bool from_input = false;
  int rslot;
  if (pending != nullptr && b == N - 1) {
    from_input = true;
    rslot = -1;
    krow = kn;
  } else {
    rslot = (pending != nullptr && D <= 1) ? window_slot(b, S, W) : r.bslot;
    krow = kv + static_cast<size_t>(rslot) * (2 * a.d);
  }
  const T* vrow = from_input ? vn : krow + a.d;
  float sb;
  if (a.flags & FLAG_EXTERNAL_SCORES) {
    sb = from_input ? ext_new : score[rslot];
  } else {
    const int h = u % a.Hkv;
    sb = mlp_score_warp<T>(krow, vrow, a.d, head_w1(a, h), head_b1(a, h), head_w2(a, h), a.b2[h], a.hidden);
  }
  sb = ranking_priority(a, u, N, sb);   // b becomes eligible at step b + W + D = N
  r.sb = sb;
  if ((a.flags & FLAG_DEBUG_CHECKS) && lane == 0) {
    if (!from_input && pos[rslot] != b) set_error(a.err, DEVERR_STATE_MISMATCH);
    if (sb != sb) set_error(a.err, DEVERR_NAN_SCORE);
  }
  longrange_decide(a, u, ntk, pending, sb, b, r);
  return r;
}

// The decode kernel's deciders take the next step's decision in two halves,
// so that a unit's merge (which commits this step's row moves) need not wait
// for the next decision's scorer and argmin.  decide_load reads what the
// commit can overwrite -- the next boundary token's row, or its caller score
// -- into registers; decide_finish scores it and runs the argmin, whose only
// slot the commit changes (the pending target) counts with the pending key.
// With team_threads > 0 the warps of a deciding team meet at kDecideBar once
// each holds what it read, before their lead lets the merge commit.
// Named barrier of a CTA's decider warps when they decide one unit together.
constexpr int kDecideBar = 1;
__device__ __forceinline__ void team_bar_sync(int nthreads) {
  asm volatile("bar.sync %0, %1;" :: "r"(kDecideBar), "r"(nthreads) : "memory");
}

template <int DH>
struct DecideInput {
  double x[2 * DH / 32];   // this lane's scorer inputs
  float sext;              // caller score
  int b;                   // boundary token position, -1: none
};

template <typename T, int DH>
__device__ __noinline__ void decide_load(const LayerArgs& a, int u, int N, const T* kn, const T* vn, float ext_new,
                                         DecideInput<DH>& in, int team_threads) {
  const int lane = threadIdx.x & 31;
  const int S = a.S, W = a.W, D = a.D, NS = a.NS;
  const int b = N - W - D;
  in.b = -1;
  in.sext = 0.f;
  if (b < S) {
    if (team_threads > 0) team_bar_sync(team_threads);
    return;
  }
  in.b = b;
  // before the pending commit: b is the token appended by that step (W = 1,
  // D = 0), or still in its window slot (D <= 1), or in its staging slot
  const bool from_input = (b == N - 1);
  const int rslot = from_input ? -1 : (D <= 1 ? window_slot(b, S, W) : staging_slot(b, S, W, D));
  const T* kv = reinterpret_cast<const T*>(a.kv + static_cast<size_t>(u) * NS * a.row_bytes);
  const T* krow = from_input ? kn : kv + static_cast<size_t>(rslot) * (2 * DH);
  const T* vrow = from_input ? vn : krow + DH;
  if (a.flags & FLAG_EXTERNAL_SCORES)
    in.sext = from_input ? ext_new : a.score[static_cast<size_t>(u) * NS + rslot];
  else
    load_scorer_input<T, 2 * DH>(krow, vrow, in.x);
  if ((a.flags & FLAG_DEBUG_CHECKS) && lane == 0 && !from_input && a.pos[static_cast<size_t>(u) * NS + rslot] != b)
    set_error(a.err, DEVERR_STATE_MISMATCH);
  if (team_threads > 0) team_bar_sync(team_threads);
}

// decide_finish: the decision from what decide_load read, taken by one warp
// (nteam = 1) or by the nteam decider warps of a CTA together (team index
// dw), in launches where each CTA decides one unit at most.  Warp dw forms
// the MLP terms of the hidden blocks [dw nb / nteam, (dw + 1) nb / nteam)
// (nb = hidden / 16) and scans the dw-th of nteam equal parts of the
// long-range keys, so a team pays one round trip of loads for each of the
// two steps instead of several.  The parts meet in shared memory (named
// barrier kDecideBar over the team): the MLP parts are summed in team order
// and the partial minima compared (keys are unique), and every warp returns
// the same decision.  A team sums the score's fp64 terms in another order
// than one warp does; both round once to fp32.
struct DecideTeam {
  double part;
  unsigned long long best;
  int slot, pad;
};
static_assert(sizeof(DecideTeam) == 24, "team slot size");


template <int DH>
__device__ __noinline__ Decision decide_finish(const LayerArgs& a, int u, int N, int ntk, const Decision* pending,
                                               const DecideInput<DH>& in, int dw, int nteam, DecideTeam* team) {
  Decision r;
  r.p = N; r.bpos = -1; r.bslot = -1; r.tgt = -1; r.evict = -1; r.sb = 0.f; r.pad[0] = r.pad[1] = 0;
  if (in.b < 0) return r;   // the same in every warp of a team
  const int lane = threadIdx.x & 31;
  const int S = a.S, W = a.W, D = a.D, K = a.K;
  const int b = in.b;
  r.bpos = b;
  r.bslot = (D == 0) ? window_slot(b, S, W) : staging_slot(b, S, W, D);
  float sb;
  if (a.flags & FLAG_EXTERNAL_SCORES) {
    sb = in.sext;
  } else {
    const int h = u % a.Hkv;
    const float* w1 = head_w1(a, h);
    if (a.hidden == 0) {
      sb = linear_score_x<2 * DH>(in.x, w1, a.b2[h]);
    } else {
      const int nb = a.hidden / 16;
      const int j0 = 16 * (dw * nb / nteam), j1 = 16 * ((dw + 1) * nb / nteam);
      double part;
      if (a.hidden == 32) part = mlp_part_x<2 * DH, 32>(in.x, w1, head_b1(a, h), head_w2(a, h), j0, j1);
      else if (a.hidden == 64) part = mlp_part_x<2 * DH, 64>(in.x, w1, head_b1(a, h), head_w2(a, h), j0, j1);
      else part = mlp_part_x<2 * DH, 128>(in.x, w1, head_b1(a, h), head_w2(a, h), j0, j1);
      if (nteam > 1) {
        if (lane == 0) team[dw].part = part;
        team_bar_sync(nteam * 32);
        part = 0.0;
        for (int t = 0; t < nteam; ++t) part += team[t].part;
      }
      sb = static_cast<float>(part + static_cast<double>(a.b2[h]));
    }
  }
  sb = ranking_priority(a, u, N, sb);   // b becomes eligible at step b + W + D = N
  r.sb = sb;
  if ((a.flags & FLAG_DEBUG_CHECKS) && dw == 0 && lane == 0 && sb != sb) set_error(a.err, DEVERR_NAN_SCORE);
  const int base = topk_base(S, W, D);
  if (ntk < K) {
    r.tgt = base + ntk;     // fill-up: next free long-range slot, nobody leaves
    r.evict = -1;
  } else if (K == 0) {
    r.evict = r.bslot;
  } else {
    const int q = (K + nteam - 1) / nteam;
    int mslot;
    uint64_t best = longrange_min(a, u, pending, min(K, dw * q), min(K, (dw + 1) * q), mslot);
    if (nteam > 1) {
      if (lane == 0) {
        team[dw].best = best;
        team[dw].slot = mslot;
      }
      team_bar_sync(nteam * 32);
      best = ~0ull;
      for (int t = 0; t < nteam; ++t) {
        const uint64_t k = team[t].best;
        if (k < best) { best = k; mslot = team[t].slot; }
      }
    }
    if (rank_key(sb, b) > best) {
      r.tgt = mslot;
      r.evict = mslot;
    } else {
      r.evict = r.bslot;
    }
  }
  if (nteam > 1) team_bar_sync(nteam * 32);   // every warp has read the slots: free for the next unit
  return r;
}

// Commit of the step appending token N for unit u (one warp): moves rows as
// the decision says, writes the new token, updates the unit's counters.
template <typename T>
__device__ void commit_warp(const LayerArgs& a, int u, int N, int ntk_after, const Decision& r, const T* kn,
                            const T* vn, float ext_new) {
  const int lane = threadIdx.x & 31;
  const int S = a.S, W = a.W, D = a.D, NS = a.NS, RB = a.row_bytes;
  uint8_t* kv = a.kv + static_cast<size_t>(u) * NS * RB;
  int32_t* pos = a.pos + static_cast<size_t>(u) * NS;
  float* score = a.score + static_cast<size_t>(u) * NS;
  if ((a.flags & FLAG_DEBUG_CHECKS) && lane == 0) {
    if (r.p != N) set_error(a.err, DEVERR_STATE_MISMATCH);
    if (r.bpos >= 0 && pos[r.bslot] != r.bpos) set_error(a.err, DEVERR_STATE_MISMATCH);
  }
  const int p = N;
  const int ns = p < S ? p : window_slot(p, S, W);
  const int o = (p >= S && p - W >= S) ? p - W : -1;
  const int st = (D > 0 && o >= 0) ? staging_slot(o, S, W, D) : -1;
  const int half = a.d * static_cast<int>(sizeof(T));
  // Read every source row first (one round trip), then write: the moves are
  // tgt <- bslot, st <- ns, ns <- new, and bslot may equal st.
  constexpr int kMaxChunks = 2;   // 16-byte chunks per lane per row (rows <= 1024 bytes)
  uint4 rb[kMaxChunks], rn[kMaxChunks], rw[kMaxChunks];
#pragma unroll
  for (int t = 0; t < kMaxChunks; ++t) {
    const int i = (lane + 32 * t) * 16;
    if (i < RB) {
      if (r.tgt >= 0) rb[t] = *reinterpret_cast<const uint4*>(kv + static_cast<size_t>(r.bslot) * RB + i);
      if (st >= 0) rn[t] = *reinterpret_cast<const uint4*>(kv + static_cast<size_t>(ns) * RB + i);
      rw[t] = (i < half) ? *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(kn) + i)
                         : *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vn) + (i - half));
    }
  }
  const float sns = (st >= 0) ? score[ns] : 0.f;
  __syncwarp();
#pragma unroll
  for (int t = 0; t < kMaxChunks; ++t) {
    const int i = (lane + 32 * t) * 16;
    if (i < RB) {
      if (r.tgt >= 0) *reinterpret_cast<uint4*>(kv + static_cast<size_t>(r.tgt) * RB + i) = rb[t];
      if (st >= 0) *reinterpret_cast<uint4*>(kv + static_cast<size_t>(st) * RB + i) = rn[t];
      *reinterpret_cast<uint4*>(kv + static_cast<size_t>(ns) * RB + i) = rw[t];
    }
  }
  if (lane == 0) {
    if (r.tgt >= 0) { pos[r.tgt] = r.bpos; score[r.tgt] = r.sb; }
    if (st >= 0) { pos[st] = o; score[st] = sns; }
    pos[ns] = p;
    score[ns] = (a.flags & FLAG_EXTERNAL_SCORES) ? ext_new : 0.f;
    a.state[4 * u + 0] = p + 1;
    a.state[4 * u + 1] = ntk_after;
  }
  __syncwarp();
}

// Merge the split-K partials of a unit, write the output, and (in a step)
// commit the step's row moves: boundary token into its long-range slot,
// window token into the staging ring, new token into its window slot.  Run by
// one warp once every contributor of the unit has arrived.  Two dependent
// round trips: (1) every segment's (m, l) and the step's decision; (2) every
// segment's accumulators and the rows the commit moves.  The new token was
// already folded into the first partial.
template <typename T, int DH, int G>
__device__ __noinline__ void merge_unit(const LayerArgs& a, const DecodeScratch& sc, bool step, int N, int ntk_after,
                                        int64_t unit, int nseg, const T* __restrict__ k_new,
                                        const T* __restrict__ v_new, const float* __restrict__ ext,
                                        T* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  constexpr int DPL = DH / 32;   // output dims per lane (contiguous)
  static_assert(DPL == 2 || DPL == 4, "head_dim 64 or 128");
  const float* pm = sc.part_ml + unit * kMaxSeg * (G * 2);
  const float* pa = sc.part_acc + unit * kMaxSeg * (G * DH);
  T* ou = out + unit * (G * DH);
  const int S = a.S, W = a.W, D = a.D, NS = a.NS, RB = a.row_bytes;

  // ---- one round trip: every load below is issued before any result is used.
  // segment maxima/sums (lane s holds segments s, s + 32), the decision, the
  // rows the commit moves (their slots follow from N alone: the boundary
  // token's row is read even when it is dropped), and the accumulators of the
  // first kSB segments.
  float mlA[2 * G], mlB[2 * G];
#pragma unroll
  for (int t = 0; t < 2 * G; ++t) {
    mlA[t] = (lane < nseg) ? __ldcg(pm + lane * G * 2 + t) : 0.f;
    mlB[t] = (lane + 32 < nseg) ? __ldcg(pm + (lane + 32) * G * 2 + t) : 0.f;
  }
  Decision r;
  r.tgt = -1; r.bslot = -1; r.bpos = -1; r.p = N; r.evict = -1; r.sb = 0.f;
  if (step) r = a.dec[static_cast<size_t>(N & 1) * a.units + unit];
  const int p = N;
  const int ns = p < S ? p : window_slot(p, S, W);
  const int o = (p >= S && p - W >= S) ? p - W : -1;
  const int st = (D > 0 && o >= 0) ? staging_slot(o, S, W, D) : -1;
  const int bb = N - W - D;   // boundary token of this step
  const int bslot = (bb >= S) ? ((D == 0) ? window_slot(bb, S, W) : staging_slot(bb, S, W, D)) : -1;
  uint8_t* kv = a.kv + static_cast<size_t>(unit) * NS * RB;
  int32_t* pos = a.pos + static_cast<size_t>(unit) * NS;
  float* score = a.score + static_cast<size_t>(unit) * NS;
  const int half = DH * static_cast<int>(sizeof(T));
  constexpr int kMaxChunks = 2;   // 16-byte chunks per lane per row (rows <= 1024 bytes)
  uint4 rb[kMaxChunks], rn[kMaxChunks], rw[kMaxChunks];
  float sns = 0.f;
  if (step) {
#pragma unroll
    for (int t = 0; t < kMaxChunks; ++t) {
      const int i = (lane + 32 * t) * 16;
      if (i < RB) {
        if (bslot >= 0) rb[t] = *reinterpret_cast<const uint4*>(kv + static_cast<size_t>(bslot) * RB + i);
        if (st >= 0) rn[t] = *reinterpret_cast<const uint4*>(kv + static_cast<size_t>(ns) * RB + i);
        rw[t] = (i < half) ? *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(k_new + unit * DH) + i)
                           : *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(v_new + unit * DH) +
                                                             (i - half));
      }
    }
    if (st >= 0) sns = score[ns];
  }
  constexpr int kSB = 4;   // segments per batch of accumulator loads
  float pv[kSB][G][DPL];
  auto load_batch = [&](int s0) {
#pragma unroll
    for (int t = 0; t < kSB; ++t) {
      if (s0 + t < nseg) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float* src = pa + (s0 + t) * G * DH + g * DH + lane * DPL;
          if constexpr (DPL == 4) {
            const float4 v4 = __ldcg(reinterpret_cast<const float4*>(src));
            pv[t][g][0] = v4.x; pv[t][g][1] = v4.y; pv[t][g][2] = v4.z; pv[t][g][3] = v4.w;
          } else {
            const float2 v2 = __ldcg(reinterpret_cast<const float2*>(src));
            pv[t][g][0] = v2.x; pv[t][g][1] = v2.y;
          }
        }
      }
    }
  };
  load_batch(0);

  float M[G], L[G], wA[G], wB[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float ma = (lane < nseg) ? mlA[2 * g] : kNegInf;
    const float mb = (lane + 32 < nseg) ? mlB[2 * g] : kNegInf;
    float mx = fmaxf(ma, mb);
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
    M[g] = mx;
    wA[g] = (ma != kNegInf) ? fast_exp2(ma - mx) : 0.f;
    wB[g] = (mb != kNegInf) ? fast_exp2(mb - mx) : 0.f;
    float ls = wA[g] * mlA[2 * g + 1] + wB[g] * mlB[2 * g + 1];
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o2);
    L[g] = ls;
  }

  float o_acc[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < DPL; ++e) o_acc[g][e] = 0.f;
  for (int s0 = 0; s0 < nseg; s0 += kSB) {
    if (s0 > 0) load_batch(s0);
#pragma unroll
    for (int t = 0; t < kSB; ++t) {
      const int sI = s0 + t;
      if (sI < nseg) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float wsv = __shfl_sync(0xffffffffu, sI < 32 ? wA[g] : wB[g], sI & 31);
#pragma unroll
          for (int e = 0; e < DPL; ++e) o_acc[g][e] = fmaf(pv[t][g][e], wsv, o_acc[g][e]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float inv = L[g] > 0.f ? 1.f / L[g] : 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) ou[g * DH + lane * DPL + e] = Elem<T>::from_f32(o_acc[g][e] * inv);
  }
  if (!step) return;
  if ((a.flags & FLAG_DEBUG_CHECKS) && lane == 0) {
    if (r.p != N) set_error(a.err, DEVERR_STATE_MISMATCH);
    if (r.bpos >= 0 && pos[r.bslot] != r.bpos) set_error(a.err, DEVERR_STATE_MISMATCH);
    if (r.tgt >= 0 && r.bslot != bslot) set_error(a.err, DEVERR_STATE_MISMATCH);
  }
  __syncwarp();
#pragma unroll
  for (int t = 0; t < kMaxChunks; ++t) {
    const int i = (lane + 32 * t) * 16;
    if (i < RB) {
      if (r.tgt >= 0 && bslot >= 0) *reinterpret_cast<uint4*>(kv + static_cast<size_t>(r.tgt) * RB + i) = rb[t];
      if (st >= 0) *reinterpret_cast<uint4*>(kv + static_cast<size_t>(st) * RB + i) = rn[t];
      *reinterpret_cast<uint4*>(kv + static_cast<size_t>(ns) * RB + i) = rw[t];
    }
  }
  if (lane == 0) {
    if (r.tgt >= 0) { pos[r.tgt] = r.bpos; score[r.tgt] = r.sb; }
    if (st >= 0) { pos[st] = o; score[st] = sns; }
    pos[ns] = p;
    score[ns] = (a.flags & FLAG_EXTERNAL_SCORES) ? ext[unit] : 0.f;
    a.state[4 * unit + 0] = p + 1;
    a.state[4 * unit + 1] = ntk_after;
  }
  __syncwarp();
}

// Before the kernel waits for its predecessor in the stream: warm L2 with
// what this warp reads first, so the HBM idles less across the launch
// boundary.  Only L2 prefetches are issued (hints: nothing is read into the
// SM); the layer counters read here may be stale when the predecessor is a
// launch of this same layer, so they only choose addresses, each clamped to
// its array.  Consumer warps: the first kPrefetchTiles tiles of their range.
// Decider warps: the long-range keys and candidate boundary rows of their
// units, and (one CTA per KV head) that head's scorer weights.
template <int NCW, int NDW>
__device__ __forceinline__ void l2_warmup(const LayerArgs& a, bool step, int warp, int lane) {
  if (lane != 0) return;
  const int N = ld_relaxed(&a.layer->n_seen);
  const int ntk = ld_relaxed(&a.layer->n_topk);
  const int S = a.S, W = a.W, D = a.D, K = a.K, NS = a.NS;
  if (N < 1 || N > a.max_context || ntk < 0 || ntk > K) return;
  const int64_t rb = a.row_bytes;
  if (warp < NCW) {
    if (kPrefetchTiles == 0) return;
    const int tpu = (S + W + D + ntk + TS - 1) / TS;
    const int64_t total = static_cast<int64_t>(a.units) * tpu;
    const int64_t nw = decode_active_warps(total, tpu, static_cast<int64_t>(gridDim.x) * NCW);
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * NCW + warp;
    if (gw >= nw) return;
    const int64_t lo = seg_lo(gw, total, nw);
    const int64_t cnt = seg_lo(gw + 1, total, nw) - lo;
    for (int i = 0; i < kPrefetchTiles && i < cnt; ++i) {
      const int64_t t = lo + i;
      const int64_t u = t / tpu;
      const int jt = static_cast<int>(t - u * tpu);
      const int rows = min(TS, NS - jt * TS);
      if (rows > 0) prefetch_l2(a.kv + (u * NS + static_cast<int64_t>(jt) * TS) * rb, static_cast<uint32_t>(rows * rb));
    }
    return;
  }
  if (!step) return;
  const int dw = warp - NCW;
  const int base = topk_base(S, W, D);
  const int b = N + 1 - W - D;   // boundary token of the decision taken in this launch
  for (int u = blockIdx.x * NDW + dw; u < a.units; u += gridDim.x * NDW) {
    if (K > 0) {
      // [lo, hi) byte range of the unit's long-range scores / positions, in 16-byte units
      const int64_t lo = (static_cast<int64_t>(u) * NS + base) * 4 / 16 * 16;
      const int64_t hi = (static_cast<int64_t>(u) * NS + base + K) * 4 / 16 * 16;
      if (hi > lo) {
        prefetch_l2(reinterpret_cast<const uint8_t*>(a.score) + lo, static_cast<uint32_t>(hi - lo));
        prefetch_l2(reinterpret_cast<const uint8_t*>(a.pos) + lo, static_cast<uint32_t>(hi - lo));
      }
    }
    if (b >= S && b < N) {
      const uint8_t* ur = a.kv + static_cast<int64_t>(u) * NS * rb;
      prefetch_l2(ur + static_cast<int64_t>(window_slot(b, S, W)) * rb, static_cast<uint32_t>(rb));
      if (D > 0) prefetch_l2(ur + static_cast<int64_t>(staging_slot(b, S, W, D)) * rb, static_cast<uint32_t>(rb));
    }
  }
  if (dw == 0 && blockIdx.x < a.Hkv && !(a.flags & FLAG_EXTERNAL_SCORES) && a.w1 != nullptr) {
    const float* w1 = head_w1(a, blockIdx.x);
    if ((reinterpret_cast<uintptr_t>(w1) & 15u) == 0)
      prefetch_l2(w1, static_cast<uint32_t>(a.hidden > 0 ? a.hidden : 1) * 2 * a.d * 4);
  }
}

template <typename T, int DH, int G, int NCW, int NSTG, int NDW>
__global__ void __launch_bounds__((NCW + NDW) * 32, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ LayerArgs a,
              const __grid_constant__ DecodeScratch sc, const int mode, const T* __restrict__ q,
              const T* __restrict__ k_new, const T* __restrict__ v_new, const float* __restrict__ ext,
              T* __restrict__ out) {
  using GE = Geo<T, DH, G>;
  using SM = Smem<T, DH, G, NCW, NSTG>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + SM::BAR);   // [NCW][NSTG]
  uint64_t* q_bar = full_bar + NCW * NSTG;                             // [NCW][2]
  int* mq = reinterpret_cast<int*>(smem + SM::MQ);                     // entries, then tail, head, done

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool step = (mode != MODE_ATTEND);

  if (threadIdx.x == 0) {
    for (int i = 0; i < NCW * (NSTG + 2); ++i) mbar_init(&full_bar[i], 1);
    mbar_fence_init();
  }
  for (int i = threadIdx.x; i < kMergeCap + 4; i += blockDim.x) mq[i] = 0;
  // Programmatic dependent launch: let the next kernel in the stream start its
  // prologue as SMs free up, and wait here until the previous one has
  // completed and its writes are visible (everything below reads its results).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  l2_warmup<NCW, NDW>(a, step, warp, lane);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __syncthreads();
  if ((smem_u32(smem) & 1023u) != 0u) {  // the swizzled boxes need 1024-byte alignment
    if (threadIdx.x == 0) set_error(a.err, DEVERR_BAD_INDEX);
    return;
  }

  const int N = a.layer->n_seen;      // the cache holds tokens 0..N-1
  const int ntk = a.layer->n_topk;
  const int S = a.S, W = a.W, D = a.D, K = a.K;
  if (step && N >= a.max_context) {
    if (threadIdx.x == 0) set_error(a.err, DEVERR_CONTEXT_OVERFLOW);
    return;
  }
  const int ntk_after = ntk + ((step && N - W - D >= S && ntk < K) ? 1 : 0);
  ValidGeom vg;
  vg.p = N - 1; vg.S = S; vg.W = W; vg.D = D;
  vg.nse = S + W + D + ntk;
  vg.full = N >= S + W + D;
  const int tpu = (vg.nse + TS - 1) / TS;
  const int64_t total = static_cast<int64_t>(a.units) * tpu;
  const int64_t nw = decode_active_warps(total, tpu, static_cast<int64_t>(gridDim.x) * NCW);
  const float qscale = kLog2e * rsqrtf(static_cast<float>(DH));

  auto nseg_of = [&](int64_t unit) -> int {
    return static_cast<int>(warp_of_tile(unit * tpu + tpu - 1, total, nw) - warp_of_tile(unit * tpu, total, nw) + 1);
  };
  auto do_merge = [&](int64_t unit) {
    merge_unit<T, DH, G>(a, sc, step, N, ntk_after, unit, nseg_of(unit), k_new, v_new, ext, out);
    __syncwarp();
    if (lane == 0) sc.ticket[unit] = 0;
  };
  // Queue a unit whose contributors have all arrived, for this CTA's merge
  // helpers: a ring of kMergeCap entries (0 = empty, else unit + 1) followed
  // by its tail counter.  The pusher claims a slot, then fills its entry once
  // the helper that took the previous value there has emptied it (bounded
  // wait); helpers take entries by exchange with 0, so every value is taken
  // once.  If the wait gives up, the unit is dropped: the error word reports
  // the timeout and the step's outputs are undefined.
  auto push_merge = [&](int64_t unit) {
    if (lane == 0) {
      const int slot = atomicAdd(&mq[kMergeCap], 1);
      const uint64_t t0 = global_ns();
      while (atomicCAS(&mq[slot % kMergeCap], 0, static_cast<int>(unit) + 1) != 0) {
        if (global_ns() - t0 > kMergeWaitLimitNs) { set_error(a.err, DEVERR_TIMEOUT); break; }
        __nanosleep(64);
      }
    }
    __syncwarp();
  };
  // Count one finished contributor of `unit`; returns the previous count (lane 0's
  // value in every lane).  The caller pushes the merge if it was the last.
  auto arrive = [&](int64_t unit) -> int {
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = ticket_add(&sc.ticket[unit]);
    return prev;
  };
  auto need_of = [&](int64_t unit) -> int { return nseg_of(unit) + (step ? 1 : 0); };
  // Pop queued merges until every consumer warp of the CTA has finished and
  // the queue is drained (bounded wait; all traffic is this CTA's shared memory).
  auto help = [&]() {
    const uint64_t t0 = global_ns();
    while (true) {
      int got = -1;
      if (lane == 0) {
        const int tail = atomicAdd(&mq[kMergeCap], 0);
        const int head = atomicAdd(&mq[kMergeCap + 1], 0);
        if (head < tail) {
          if (atomicCAS(&mq[kMergeCap + 1], head, head + 1) == head) {
            int v;
            while ((v = atomicExch(&mq[head % kMergeCap], 0)) == 0) {
              if (global_ns() - t0 > kMergeWaitLimitNs) break;
            }
            got = v > 0 ? v - 1 : -3;
          }
        } else if (atomicAdd(&mq[kMergeCap + 2], 0) == NCW) {
          __threadfence_block();
          if (head >= atomicAdd(&mq[kMergeCap], 0)) got = -2;
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      if (got == -2) break;
      if (got == -3) {
        if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
        break;
      }
      if (got >= 0) {
        __threadfence();
        do_merge(got);
        continue;
      }
      if (global_ns() - t0 > kMergeWaitLimitNs) {
        if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
        break;
      }
      __nanosleep(256);
    }
  };
  auto consumer_done = [&]() {
    __syncwarp();
#ifdef KVPOP_TEST_HOOKS
    if (a.test_hook == TEST_HOOK_WITHHOLD_DONE && blockIdx.x == 0 && warp == 0) return;
#endif
    if (lane == 0) {
      __threadfence_block();
      atomicAdd(&mq[kMergeCap + 2], 1);
    }
    __syncwarp();
  };
  // Every warp of a step launch reports here once; the last one advances the
  // layer counters (nobody reads them again in this launch).
  auto finish_launch = [&]() {
    if (!step) return;
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      const int prev = atomicAdd(&a.layer->ticket, 1);
      if (prev == static_cast<int>(gridDim.x) * (NCW + NDW) - 1) {
        a.layer->n_seen = N + 1;
        a.layer->n_topk = ntk_after;
        a.layer->ticket = 0;
        __threadfence();
      }
    }
  };

  if (warp >= NCW) {
    // ---------------- deciders, then merge helpers ----------------
    static_assert(NDW <= kMaxDeciders, "team slots");
    if (step) {
      const int dw = warp - NCW;
      // with at most one unit per CTA, the CTA's decider warps take it together
      const bool team = a.units <= static_cast<int>(gridDim.x);
      const bool lead = !team || dw == 0;   // the warp that arrives and stores the decision
      DecideTeam* team_sm = reinterpret_cast<DecideTeam*>(smem + SM::TEAM);
      for (int u = team ? blockIdx.x : blockIdx.x * NDW + dw; u < a.units;
           u += team ? gridDim.x : gridDim.x * NDW) {
        if (mode == MODE_STEP) {   // MODE_STEP_NODECIDE: the next step's kernel decides
          const Decision cur = a.dec[static_cast<size_t>(N & 1) * a.units + u];
          DecideInput<DH> din;
          decide_load<T, DH>(a, u, N + 1, k_new + static_cast<size_t>(u) * DH, v_new + static_cast<size_t>(u) * DH,
                             ext ? ext[u] : 0.f, din, team ? NDW * 32 : 0);
          if (lead) {
            const int prev = __shfl_sync(0xffffffffu, arrive(u), 0);
            if (prev == need_of(u) - 1) push_merge(u);
          }
          const Decision nx = decide_finish<DH>(a, u, N + 1, ntk_after, &cur, din, team ? dw : 0, team ? NDW : 1,
                                                team_sm);
          if (lead && lane == 0) a.dec[static_cast<size_t>((N + 1) & 1) * a.units + u] = nx;
          continue;
        }
        if (lead) {
          const int prev = __shfl_sync(0xffffffffu, arrive(u), 0);
          if (prev == need_of(u) - 1) push_merge(u);
        }
      }
    }
    help();
    finish_launch();
    return;
  }

  // ---------------- consumers ----------------
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * NCW + warp;
  if (gw >= nw) {
    consumer_done();
    help();
    finish_launch();
    return;
  }
  const int64_t lo = seg_lo(gw, total, nw);
  const int cnt = static_cast<int>(seg_lo(gw + 1, total, nw) - lo);
  const int last_unit = static_cast<int>((lo + cnt - 1) / tpu);
  uint8_t* ring = smem + SM::RINGS + warp * NSTG * GE::STAGE;
  uint8_t* qsm = smem + SM::Q + warp * GE::QBYTES;
  uint8_t* psm = smem + SM::P + warp * GE::PBYTES;
  uint8_t* qraw = smem + SM::QRAW + warp * 2 * SM::QRB;
  uint64_t* fb = full_bar + warp * NSTG;
  uint64_t* qb = q_bar + warp * 2;
  const int NS = a.NS;

  // q (and in a step the new token's k, v) of a unit -> raw buffer `buf`
  auto issue_q = [&](int unit, int buf) {
    constexpr uint32_t kq = G * DH * GE::ESZ, kr = DH * GE::ESZ;
    if (lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&qb[buf], kq + (step ? 2 * kr + 32 : 0));
      uint8_t* dst = qraw + buf * SM::QRB;
      bulk_g2s(dst, q + static_cast<int64_t>(unit) * (G * DH), kq, &qb[buf]);
      if (step) {
        bulk_g2s(dst + kq, k_new + static_cast<int64_t>(unit) * DH, kr, &qb[buf]);
        bulk_g2s(dst + kq + kr, v_new + static_cast<int64_t>(unit) * DH, kr, &qb[buf]);
        bulk_g2s(dst + kq + 2 * kr, a.dec + static_cast<size_t>(N & 1) * a.units + unit, 32, &qb[buf]);
      }
    }
  };

  // issue cursor (tile index within the range -> unit, tile of the unit)
  int iu = static_cast<int>(lo / tpu), ij = static_cast<int>(lo - static_cast<int64_t>(iu) * tpu);
  int istage = 0;
  auto issue_next = [&]() {
    if (lane == 0) mbar_arrive_expect_tx(&fb[istage], GE::STAGE);
    __syncwarp();
    if (lane < GE::NBLK)
      tma_load_2d(ring + istage * GE::STAGE + lane * GE::BOX, &tmap, lane * GE::BOXELEMS, iu * NS + ij * TS,
                  &fb[istage]);
    if (++ij == tpu) { ij = 0; ++iu; }
    if (++istage == NSTG) istage = 0;
  };
  // last finished segment and its ticket result, checked one segment later
  int pend_unit = -1, pend_prev = 0;
  auto check_pending = [&]() {
    if (pend_unit < 0) return;
    const int prev = __shfl_sync(0xffffffffu, pend_prev, 0);
    if (prev == need_of(pend_unit) - 1) push_merge(pend_unit);
    pend_unit = -1;
  };

  if constexpr (sizeof(T) == 2) {
    // ---- bf16: both contractions of a tile on the tensor cores ----
    // mma.sync m16n8k16, fp32 accumulate.  S = Q K^T with the G query heads
    // as the M rows (rows G..15 zero) and the tile's 16 slots as two n-blocks;
    // O^T = V^T P^T with the head dims as M (DH / 16 blocks) and the heads as
    // N, so the S fragment of a tile, rounded to bf16, is the B fragment of
    // its P V as it stands.  Lane (gid, tig) = (lane / 4, lane % 4) keeps the
    // softmax state of head gid over slots 2 tig, 2 tig + 1, 8 + 2 tig,
    // 9 + 2 tig, and O^T of heads 2 tig, 2 tig + 1 at dims 16 mb + gid and
    // 16 mb + gid + 8.  K and V fragments come from the swizzled tile by
    // ldmatrix (row addresses of 8 consecutive slots hit 8 distinct bank
    // groups).  Per tile and warp: 2 DH / 16 ldmatrix, 3 DH / 16 MMAs.
    constexpr int KS = DH / 16;
    const int gid = lane >> 2, tig = lane & 3;
    const bool hreal = gid < G;
    const int lslot = 8 * (lane >> 4) + (lane & 7);   // ldmatrix row: matrix lane / 8, row lane % 8
    const int lhalf = (lane >> 3) & 1;                // second 8-element half of the 16
    uint32_t qa[KS][2];
    float o[KS][4];
    float m_run = kNegInf, l_run = 0.f;
    int evict = -1;
    int cur = -1;
    int qbuf = 0;
    uint32_t qphase = 0;   // bit b = parity of raw buffer b's next completion

    // Start a unit segment: q into A fragments, reset the softmax state, fold
    // the new token in if this warp holds the unit's first tile, and prefetch
    // the next unit's q.
    auto start_unit = [&](int unit, bool first_tile) {
      if (!mbar_wait(&qb[qbuf], (qphase >> qbuf) & 1u)) {
        if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
      }
      qphase ^= 1u << qbuf;
      const uint8_t* raw = qraw + qbuf * SM::QRB;
      __syncwarp();
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(raw);   // q as bf16 pairs, [G][DH / 2]
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qa[ks][0] = hreal ? qw[(gid * DH + ks * 16 + 2 * tig) >> 1] : 0u;
        qa[ks][1] = hreal ? qw[(gid * DH + ks * 16 + 8 + 2 * tig) >> 1] : 0u;
      }
      evict = step ? reinterpret_cast<const Decision*>(raw + G * DH * GE::ESZ + 2 * DH * GE::ESZ)->evict : -1;
      m_run = kNegInf;
      l_run = 0.f;
#pragma unroll
      for (int mb = 0; mb < KS; ++mb)
#pragma unroll
        for (int r = 0; r < 4; ++r) o[mb][r] = 0.f;
      if (step && first_tile) {
        // the appended token: score q . k_new and take it as the first slot
        constexpr int DPL = DH / 32;
        const T* qr = reinterpret_cast<const T*>(raw);
        const T* kn = qr + G * DH;
        const T* vn = kn + DH;
        float mnew = kNegInf;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float part = 0.f;
#pragma unroll
          for (int e = 0; e < DPL; ++e)
            part = fmaf(Elem<T>::to_f32(qr[g * DH + lane * DPL + e]), Elem<T>::to_f32(kn[lane * DPL + e]), part);
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o2);
          if (g == gid) mnew = part * qscale;   // p = exp2(s - m) = 1
        }
        m_run = mnew;
        l_run = (hreal && tig == 0) ? 1.f : 0.f;
#pragma unroll
        for (int mb = 0; mb < KS; ++mb) {
          const float v0 = Elem<T>::to_f32(vn[16 * mb + gid]);
          const float v1 = Elem<T>::to_f32(vn[16 * mb + gid + 8]);
          o[mb][0] = v0; o[mb][1] = v0; o[mb][2] = v1; o[mb][3] = v1;
        }
      }
      __syncwarp();
      if (unit < last_unit) issue_q(unit + 1, qbuf ^ 1);
      qbuf ^= 1;
    };

    auto finalize = [&](int unit) {
      float l = l_run;
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const int64_t first = warp_of_tile(static_cast<int64_t>(unit) * tpu, total, nw);
      const int seg = static_cast<int>(gw - first);
      if (seg >= kMaxSeg) {  // cannot happen: the split bounds the segments per unit
        if (lane == 0) set_error(a.err, DEVERR_BAD_INDEX);
        return;
      }
      float* pa = sc.part_acc + (static_cast<int64_t>(unit) * kMaxSeg + seg) * (G * DH);
      float* pmv = sc.part_ml + (static_cast<int64_t>(unit) * kMaxSeg + seg) * (G * 2);
#pragma unroll
      for (int mb = 0; mb < KS; ++mb)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int hh = 2 * tig + (r & 1);
          if (hh < G) pa[hh * DH + 16 * mb + gid + 8 * (r >> 1)] = o[mb][r];
        }
      if (tig == 0 && hreal) {
        pmv[2 * gid] = m_run;
        pmv[2 * gid + 1] = l;
      }
      pend_unit = unit;
      pend_prev = arrive(unit);   // checked later, so the atomic's round trip overlaps streaming
    };

    // consume cursor
    int cu = static_cast<int>(lo / tpu), cj = static_cast<int>(lo - static_cast<int64_t>(cu) * tpu);
    // first unit's q before the tile burst (it would queue behind it otherwise)
    issue_q(cu, 0);
    {
      const int npre = cnt < NSTG ? cnt : NSTG;
      for (int i = 0; i < npre; ++i) issue_next();
    }
    int cstage = 0;
    uint32_t cphase = 0;
    bool failed = false;
    int failed_at = -1;
    for (int i = 0; i < cnt; ++i) {
      const int s0 = cj * TS;
      if (cu != cur) {
        if (cur >= 0) {
          check_pending();
          finalize(cur);
        }
        cur = cu;
        start_unit(cu, cj == 0);
      }
      if (!mbar_wait(&fb[cstage], cphase)) {
        if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
        failed = true;
        failed_at = i;
        break;
      }
      uint8_t* tile = ring + cstage * GE::STAGE;
      const uint32_t tb = smem_u32(tile);

      // ---- S = Q K^T ----
      float sacc[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int r = 0; r < 4; ++r) sacc[nb][r] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t kb[4];
        ldsm_x4(tb + GE::off(lslot, 2 * ks + lhalf), kb);
        const uint32_t qf[4] = {qa[ks][0], 0u, qa[ks][1], 0u};
        mma_bf16_16816(sacc[0], qf, kb[0], kb[1]);
        mma_bf16_16816(sacc[1], qf, kb[2], kb[3]);
      }
      float sv[4] = {sacc[0][0], sacc[0][1], sacc[1][0], sacc[1][1]};

      // Slot validity: a tile of occupied slots without the evicted one (the
      // common case) needs no per-slot test.  Rows of slots that hold no
      // token may hold anything: their V rows are zeroed so that a weight of
      // 0 cannot meet a non-finite value in the P V product (K rows need
      // nothing: their scores are replaced).
      if (!(vg.full && s0 + TS <= vg.nse && (evict < s0 || evict >= s0 + TS))) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int slot = s0 + 8 * (r >> 1) + 2 * tig + (r & 1);
          if (slot == evict || !vg.slot_ok(slot)) sv[r] = kNegInf;
        }
        const int zslot = s0 + (lane & 15);
        if (!vg.slot_ok(zslot)) {
#pragma unroll
          for (int cc = 0; cc < GE::NCHK / 2; ++cc)
            *reinterpret_cast<uint4*>(tile + GE::off(lane & 15, GE::NCHK + (lane >> 4) * (GE::NCHK / 2) + cc)) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
      }
      if (!hreal) {
#pragma unroll
        for (int r = 0; r < 4; ++r) sv[r] = kNegInf;
      }
      // ---- online softmax of head gid (exp2 domain, lazy rescale) ----
      float tmax = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
      const float tm = tmax * qscale;
      if (__any_sync(0xffffffffu, tm > m_run + kLazy)) {
        float alpha = 1.f;
        if (tm > m_run + kLazy) {
          alpha = (m_run == kNegInf) ? 0.f : fast_exp2(m_run - tm);
          m_run = tm;
          l_run *= alpha;
        }
        // this lane's O^T columns are heads 2 tig and 2 tig + 1 (quads 2 tig, 2 tig + 1)
        const float aa = __shfl_sync(0xffffffffu, alpha, 8 * tig);
        const float ab = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
#pragma unroll
        for (int mb = 0; mb < KS; ++mb) {
          o[mb][0] *= aa; o[mb][1] *= ab; o[mb][2] *= aa; o[mb][3] *= ab;
        }
      }
      const float nm = (m_run == kNegInf) ? 0.f : -m_run;   // masked scores give 2^-inf = 0
      float pw[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) pw[r] = fast_exp2(fmaf(sv[r], qscale, nm));
      l_run += (pw[0] + pw[1]) + (pw[2] + pw[3]);
      const uint32_t pb0 = pack_bf16(pw[0], pw[1]);   // P^T rows (slots) 2 tig, 2 tig + 1 of column (head) gid
      const uint32_t pb1 = pack_bf16(pw[2], pw[3]);   // slots 8 + 2 tig, 9 + 2 tig

      // ---- O^T += V^T P^T ----
#pragma unroll
      for (int mb = 0; mb < KS; ++mb) {
        uint32_t va[4];
        ldsm_x4_t(tb + GE::off(lslot, GE::NCHK + 2 * mb + lhalf), va);
        mma_bf16_16816(o[mb], va, pb0, pb1);
      }
      __syncwarp();
      if (i + NSTG < cnt) {
        fence_proxy_async_smem();
        issue_next();
      }
      if (++cj == tpu) { cj = 0; ++cu; }
      if (++cstage == NSTG) { cstage = 0; cphase ^= 1u; }
    }
    if (failed) {
      // let this warp's copies still in flight land (bounded) before it exits
      int st2 = cstage;
      uint32_t ph2 = cphase;
      for (int k2 = failed_at + 1; k2 < cnt && k2 < failed_at + NSTG; ++k2) {
        if (++st2 == NSTG) { st2 = 0; ph2 ^= 1u; }
        mbar_wait(&fb[st2], ph2);
      }
    } else if (cur >= 0) {
      check_pending();
      finalize(cur);
      check_pending();
    }
  } else {
    const int j = lane & 15;        // QK: slot of the tile
    const int h = lane >> 4;        // QK: half of the dims
    const int gq = lane / GE::LPS;  // PV: slot group
    const int c = lane % GE::LPS;   // PV: chunk of the value row

    float2 acc[G][GE::EPC / 2];
    float m[G], lp[G];
    int evict = -1;
    int cur = -1;
    int qbuf = 0;
    uint32_t qphase = 0;   // bit b = parity of raw buffer b's next completion

    // Start a unit segment: q into the fp32 layout, reset the softmax state,
    // fold the new token in if this warp holds the unit's first tile, and
    // prefetch the next unit's q.
    auto start_unit = [&](int unit, bool first_tile) {
      if (!mbar_wait(&qb[qbuf], (qphase >> qbuf) & 1u)) {
        if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
      }
      qphase ^= 1u << qbuf;
      const uint8_t* raw = qraw + qbuf * SM::QRB;
      __syncwarp();
      float* qf = reinterpret_cast<float*>(qsm);
      const T* qr = reinterpret_cast<const T*>(raw);
      for (int idx = lane; idx < G * DH; idx += 32) {
        const int g = idx / DH, dim = idx % DH;
        const int ch = dim / GE::EPC, e = dim % GE::EPC;
        const int hh = ch / GE::CH, cc = ch % GE::CH;
        qf[hh * ((GE::QHALF + 16) / 4) + (cc * G + g) * GE::EPC + e] = Elem<T>::to_f32(qr[idx]) * qscale;
      }
      evict = step ? reinterpret_cast<const Decision*>(raw + G * DH * GE::ESZ + 2 * DH * GE::ESZ)->evict : -1;
  #pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = kNegInf;
        lp[g] = 0.f;
  #pragma unroll
        for (int e = 0; e < GE::EPC / 2; ++e) acc[g][e] = make_float2(0.f, 0.f);
      }
      if (step && first_tile) {
        // the appended token: score q . k_new and take it as the first slot
        constexpr int DPL = DH / 32;
        const T* kn = reinterpret_cast<const T*>(raw + G * DH * GE::ESZ);
        const T* vn = kn + DH;
  #pragma unroll
        for (int g = 0; g < G; ++g) {
          float part = 0.f;
  #pragma unroll
          for (int e = 0; e < DPL; ++e)
            part = fmaf(Elem<T>::to_f32(qr[g * DH + lane * DPL + e]), Elem<T>::to_f32(kn[lane * DPL + e]), part);
  #pragma unroll
          for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          m[g] = part * qscale;   // p = exp2(s - m) = 1
        }
        if (lane == 0) {
  #pragma unroll
          for (int g = 0; g < G; ++g) lp[g] = 1.f;
        }
        if (gq == 0) {
          const uint4 vr = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vn) + c * 16);
          float2 v2[GE::EPC / 2];
          if constexpr (sizeof(T) == 2) {
            v2[0] = bf2_to_f2(vr.x); v2[1] = bf2_to_f2(vr.y); v2[2] = bf2_to_f2(vr.z); v2[3] = bf2_to_f2(vr.w);
          } else {
            v2[0] = make_float2(__uint_as_float(vr.x), __uint_as_float(vr.y));
            v2[1] = make_float2(__uint_as_float(vr.z), __uint_as_float(vr.w));
          }
  #pragma unroll
          for (int g = 0; g < G; ++g)
  #pragma unroll
            for (int e = 0; e < GE::EPC / 2; ++e) acc[g][e] = v2[e];
        }
      }
      __syncwarp();
      if (unit < last_unit) issue_q(unit + 1, qbuf ^ 1);
      qbuf ^= 1;
    };

    auto finalize = [&](int unit) {
      float l[G];
  #pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = lp[g];
  #pragma unroll
        for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        l[g] = v;
      }
  #pragma unroll
      for (int o = GE::LPS; o < 32; o <<= 1)
  #pragma unroll
        for (int g = 0; g < G; ++g)
  #pragma unroll
          for (int e = 0; e < GE::EPC / 2; ++e) {
            acc[g][e].x += __shfl_xor_sync(0xffffffffu, acc[g][e].x, o);
            acc[g][e].y += __shfl_xor_sync(0xffffffffu, acc[g][e].y, o);
          }
      const int64_t first = warp_of_tile(static_cast<int64_t>(unit) * tpu, total, nw);
      const int seg = static_cast<int>(gw - first);
      if (seg >= kMaxSeg) {  // cannot happen: the split bounds the segments per unit
        if (lane == 0) set_error(a.err, DEVERR_BAD_INDEX);
        return;
      }
      float* pa = sc.part_acc + (static_cast<int64_t>(unit) * kMaxSeg + seg) * (G * DH);
      float* pmv = sc.part_ml + (static_cast<int64_t>(unit) * kMaxSeg + seg) * (G * 2);
      if (lane < GE::LPS) {
  #pragma unroll
        for (int g = 0; g < G; ++g)
  #pragma unroll
          for (int e = 0; e < GE::EPC / 2; ++e)
            *reinterpret_cast<float2*>(pa + g * DH + c * GE::EPC + 2 * e) = acc[g][e];
      }
      if (lane == 0) {
  #pragma unroll
        for (int g = 0; g < G; ++g) { pmv[2 * g] = m[g]; pmv[2 * g + 1] = l[g]; }
      }
      pend_unit = unit;
      pend_prev = arrive(unit);   // checked later, so the atomic's round trip overlaps streaming
    };

    // consume cursor
    int cu = static_cast<int>(lo / tpu), cj = static_cast<int>(lo - static_cast<int64_t>(cu) * tpu);
    // first unit's q before the tile burst (it would queue behind it otherwise)
    issue_q(cu, 0);
    {
      const int npre = cnt < NSTG ? cnt : NSTG;
      for (int i = 0; i < npre; ++i) issue_next();
    }
    int cstage = 0;
    uint32_t cphase = 0;
    bool failed = false;
    int failed_at = -1;
    for (int i = 0; i < cnt; ++i) {
      const int s0 = cj * TS;
      const int nsl = min(TS, vg.nse - s0);
      if (cu != cur) {
        if (cur >= 0) {
          check_pending();
          finalize(cur);
        }
        cur = cu;
        start_unit(cu, cj == 0);
      }
      if (!mbar_wait(&fb[cstage], cphase)) {
        if (lane == 0) set_error(a.err, DEVERR_TIMEOUT);
        failed = true;
        failed_at = i;
        break;
      }
      const uint8_t* tile = ring + cstage * GE::STAGE;

      // ---- QK: lane (j, h) = slot j, dims of half h, all G heads ----
      float s[G];
      {
        float2 sa[G][2];
  #pragma unroll
        for (int g = 0; g < G; ++g) { sa[g][0] = make_float2(0.f, 0.f); sa[g][1] = make_float2(0.f, 0.f); }
        const float* qh = reinterpret_cast<const float*>(qsm + h * (GE::QHALF + 16));
  #pragma unroll
        for (int cc = 0; cc < GE::CH; ++cc) {
          const uint4 kr = *reinterpret_cast<const uint4*>(tile + GE::off(j, h * GE::CH + cc));
          float2 k2[GE::EPC / 2];
          if constexpr (sizeof(T) == 2) {
            k2[0] = bf2_to_f2(kr.x); k2[1] = bf2_to_f2(kr.y); k2[2] = bf2_to_f2(kr.z); k2[3] = bf2_to_f2(kr.w);
          } else {
            k2[0] = make_float2(__uint_as_float(kr.x), __uint_as_float(kr.y));
            k2[1] = make_float2(__uint_as_float(kr.z), __uint_as_float(kr.w));
          }
  #pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4* qp = reinterpret_cast<const float4*>(qh + (cc * G + g) * GE::EPC);
  #pragma unroll
            for (int e4 = 0; e4 < GE::EPC / 4; ++e4) {
              const float4 qv = qp[e4];
              sa[g][e4 & 1] = ffma2(make_float2(qv.x, qv.y), k2[2 * e4], sa[g][e4 & 1]);
              sa[g][e4 & 1] = ffma2(make_float2(qv.z, qv.w), k2[2 * e4 + 1], sa[g][e4 & 1]);
            }
          }
        }
  #pragma unroll
        for (int g = 0; g < G; ++g) {
          float v = (sa[g][0].x + sa[g][0].y) + (sa[g][1].x + sa[g][1].y);
          v += __shfl_xor_sync(0xffffffffu, v, 16);
          s[g] = v;
        }
      }
      // Slot validity: a tile of occupied slots without the evicted one (the
      // common case) needs no per-slot test.
      bool valid = true;
      uint32_t vmask = 0xffffu;
      if (!(vg.full && s0 + TS <= vg.nse && (evict < s0 || evict >= s0 + TS))) {
        const int slot = s0 + j;
        valid = (j < nsl) && (slot != evict) && vg.slot_ok(slot);
        vmask = __ballot_sync(0xffffffffu, valid) & 0xffffu;
      }
      // ---- online softmax (exp2 domain, lazy rescale) ----
      float sv[G];
      bool in_range = true;
  #pragma unroll
      for (int g = 0; g < G; ++g) {
        sv[g] = valid ? s[g] : kNegInf;
        in_range = in_range && (sv[g] <= m[g] + kLazy);
      }
      // The running max moves only when a tile exceeds it by 2^kLazy; one vote
      // tells whether any score of the tile does, else no tile max is needed.
      if (!__all_sync(0xffffffffu, in_range)) {
  #pragma unroll
        for (int g = 0; g < G; ++g) {
          float mt = sv[g];
  #pragma unroll
          for (int o = 1; o < 16; o <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
          if (mt > m[g] + kLazy) {   // warp-uniform
            const float alpha = (m[g] == kNegInf) ? 0.f : fast_exp2(m[g] - mt);
            m[g] = mt;
            lp[g] *= alpha;
  #pragma unroll
            for (int e = 0; e < GE::EPC / 2; ++e) {
              acc[g][e].x *= alpha;
              acc[g][e].y *= alpha;
            }
          }
        }
      }
      float p[G];
  #pragma unroll
      for (int g = 0; g < G; ++g) {
        p[g] = valid ? fast_exp2(sv[g] - m[g]) : 0.f;
        lp[g] += p[g];
      }
      if (h == 0) {
        float* pd = reinterpret_cast<float*>(psm + j * GE::PSLOT + (j / GE::SPG) * 16);
  #pragma unroll
        for (int g = 0; g < G; g += 2) {
          if (g + 1 < G)
            *reinterpret_cast<float4*>(pd + 2 * g) = make_float4(p[g], p[g], p[g + 1], p[g + 1]);
          else
            *reinterpret_cast<float2*>(pd + 2 * g) = make_float2(p[g], p[g]);
        }
      }
      __syncwarp();
      // ---- PV: lane (gq, c) = slots of group gq, value chunk c ----
      auto pv_slot = [&](int j2) {
        const float* pp = reinterpret_cast<const float*>(psm + j2 * GE::PSLOT + (j2 / GE::SPG) * 16);
        float2 pr[G];
  #pragma unroll
        for (int g = 0; g < G; g += 2) {
          if (g + 1 < G) {
            const float4 t4 = *reinterpret_cast<const float4*>(pp + 2 * g);
            pr[g] = make_float2(t4.x, t4.y);
            pr[g + 1] = make_float2(t4.z, t4.w);
          } else {
            pr[g] = *reinterpret_cast<const float2*>(pp + 2 * g);
          }
        }
        const uint4 vr = *reinterpret_cast<const uint4*>(tile + GE::off(j2, GE::NCHK + c));
        float2 v2[GE::EPC / 2];
        if constexpr (sizeof(T) == 2) {
          v2[0] = bf2_to_f2(vr.x); v2[1] = bf2_to_f2(vr.y); v2[2] = bf2_to_f2(vr.z); v2[3] = bf2_to_f2(vr.w);
        } else {
          v2[0] = make_float2(__uint_as_float(vr.x), __uint_as_float(vr.y));
          v2[1] = make_float2(__uint_as_float(vr.z), __uint_as_float(vr.w));
        }
  #pragma unroll
        for (int g = 0; g < G; ++g)
  #pragma unroll
          for (int e = 0; e < GE::EPC / 2; ++e) acc[g][e] = ffma2(pr[g], v2[e], acc[g][e]);
      };
      if (vmask == 0xffffu) {
  #pragma unroll
        for (int jj = 0; jj < GE::SPG; ++jj) pv_slot(gq * GE::SPG + jj);
      } else {
  #pragma unroll
        for (int jj = 0; jj < GE::SPG; ++jj) {
          const int j2 = gq * GE::SPG + jj;
          if ((vmask >> j2) & 1u) pv_slot(j2);
        }
      }
      __syncwarp();
      if (i + NSTG < cnt) {
        fence_proxy_async_smem();
        issue_next();
      }
      if (++cj == tpu) { cj = 0; ++cu; }
      if (++cstage == NSTG) { cstage = 0; cphase ^= 1u; }
    }
    if (failed) {
      // let this warp's copies still in flight land (bounded) before it exits
      int st2 = cstage;
      uint32_t ph2 = cphase;
      for (int k2 = failed_at + 1; k2 < cnt && k2 < failed_at + NSTG; ++k2) {
        if (++st2 == NSTG) { st2 = 0; ph2 ^= 1u; }
        mbar_wait(&fb[st2], ph2);
      }
    } else if (cur >= 0) {
      check_pending();
      finalize(cur);
      check_pending();
    }
  }
  consumer_done();
  help();
  finish_launch();
}

template <typename T>
__global__ void __launch_bounds__(128) append_kernel(const LayerArgs a, const T* __restrict__ k_new,
                                                     const T* __restrict__ v_new, const float* __restrict__ ext) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * 4 + warp;
  const int N = a.layer->n_seen;
  const int ntk = a.layer->n_topk;
  const int ntk_after = ntk + ((N - a.W - a.D >= a.S && ntk < a.K) ? 1 : 0);
  if (N >= a.max_context) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_error(a.err, DEVERR_CONTEXT_OVERFLOW);
    return;
  }
  if (u < a.units) {
    const T* kn = k_new + static_cast<size_t>(u) * a.d;
    const T* vn = v_new + static_cast<size_t>(u) * a.d;
    const float en = ext ? ext[u] : 0.f;
    const Decision r = a.dec[static_cast<size_t>(N & 1) * a.units + u];
    commit_warp<T>(a, u, N, ntk_after, r, kn, vn, en);
    __threadfence();
    __syncwarp();
    if (!a.mlstm) {   // the mLSTM scorer decides in the next step's own kernel
      const Decision nx = decide_warp<T>(a, u, N + 1, ntk_after, nullptr, kn, vn, en);
      if (lane == 0) a.dec[static_cast<size_t>((N + 1) & 1) * a.units + u] = nx;
    }
  }
  // last warp of the launch advances the layer counters
  __syncwarp();
  if (lane == 0) {
    __threadfence();
    const int prev = atomicAdd(&a.layer->ticket, 1);
    if (prev == static_cast<int>(gridDim.x) * 4 - 1) {
      a.layer->n_seen = N + 1;
      a.layer->n_topk = ntk_after;
      a.layer->ticket = 0;
      __threadfence();
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(128) decide_kernel(const LayerArgs a, int N, int ntk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * 4 + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.layer->n_seen = N;
    a.layer->n_topk = ntk;
    a.layer->ticket = 0;
  }
  if (u >= a.units) return;
  if (!a.mlstm) {   // the mLSTM scorer decides in the step's own kernel
    const Decision r = decide_warp<T>(a, u, N, ntk, nullptr, nullptr, nullptr, 0.f);
    if (lane == 0) a.dec[static_cast<size_t>(N & 1) * a.units + u] = r;
  }
  if (lane == 0) {
    a.state[4 * u + 0] = N;
    a.state[4 * u + 1] = ntk;
  }
}

template <typename T, int DH, int G>
int launch_t(const CUtensorMap& tmap, const LayerArgs& a, const DecodeScratch& sc, int mode, const void* q,
             const void* kn, const void* vn, const float* ext, void* out, int num_sms, cudaStream_t st) {
  constexpr int NCW = LaunchShape<T, G>::NCW, NSTG = LaunchShape<T, G>::NSTG, NDW = LaunchShape<T, G>::NDW;
  using SM = Smem<T, DH, G, NCW, NSTG>;
  // The shared-memory attribute belongs to the current device: set it once per
  // device (devices beyond the table get it on every call).
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev < 0 || dev >= kMaxDev || !attr_set[dev]) {
    if (cudaFuncSetAttribute(decode_kernel<T, DH, G, NCW, NSTG, NDW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SM::TOTAL) != cudaSuccess)
      return -1;
    if (dev >= 0 && dev < kMaxDev) attr_set[dev] = true;
  }
  const int64_t tpu_max = (a.NS + TS - 1) / TS;
  const int64_t total_max = static_cast<int64_t>(a.units) * tpu_max;
  int64_t grid = (total_max + NCW - 1) / NCW;
  if (grid > num_sms) grid = num_sms;
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3((NCW + NDW) * 32);
  cfg.dynamicSmemBytes = SM::TOTAL;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<T, DH, G, NCW, NSTG, NDW>, tmap, a, sc, mode,
                                           static_cast<const T*>(q), static_cast<const T*>(kn),
                                           static_cast<const T*>(vn), ext, static_cast<T*>(out));
  return e == cudaSuccess ? 0 : -1;
}

}  // namespace

namespace {
// The driver's tensor-map encoder, fetched through the runtime so that the
// library needs no link-time dependency on libcuda; null if unavailable.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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
}  // namespace

int make_decode_tensor_map(CUtensorMap* map, void* layer_kv, int dtype, int d, int64_t rows, int row_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return -1;
  const int esz = dtype == 0 ? 4 : 2;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(2 * d), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), static_cast<cuuint32_t>(TS)};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = encode(map, dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                            layer_kv, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int decode_supported(int dtype, int d, int G) {
  if (dtype == 1 && d == 128) return G == 1 || G == 2 || G == 4;
  if (d == 64) return G == 1 || G == 2 || G == 4 || G == 8;
  return 0;
}

int launch_decode(const CUtensorMap& tmap, const LayerArgs& a, int dtype, const DecodeScratch& sc, int mode,
                  const void* q, const void* k_new, const void* v_new, const float* ext_score, void* out, int num_sms,
                  cudaStream_t st) {
#define KVPOP_DISPATCH(TT, DD, GG) \
  if (a.d == DD && a.G == GG)      \
    return launch_t<TT, DD, GG>(tmap, a, sc, mode, q, k_new, v_new, ext_score, out, num_sms, st);
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

int launch_append(const LayerArgs& a, int dtype, const void* k_new, const void* v_new, const float* ext_score,
                  cudaStream_t st) {
  const int grid = (a.units + 3) / 4;
  if (dtype == 0)
    append_kernel<float><<<grid, 128, 0, st>>>(a, static_cast<const float*>(k_new),
                                               static_cast<const float*>(v_new), ext_score);
  else
    append_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(a, static_cast<const __nv_bfloat16*>(k_new),
                                                       static_cast<const __nv_bfloat16*>(v_new), ext_score);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_decide(const LayerArgs& a, int dtype, int n_seen, int n_topk, cudaStream_t st) {
  const int grid = (a.units + 3) / 4;
  if (dtype == 0)
    decide_kernel<float><<<grid, 128, 0, st>>>(a, n_seen, n_topk);
  else
    decide_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(a, n_seen, n_topk);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace kvpop
