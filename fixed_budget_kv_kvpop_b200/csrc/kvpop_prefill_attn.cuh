// Parallel sparse prefill attention under the running top-k mask (KVpop page,
// §C "Efficient Running Top-k Sparse Attention": §C.1 Mask Definition, §C.2
// Fenwick-Tree Cutoff Computation).  Host-side launch interface.
#pragma once

#include "kvpop_internal.cuh"

namespace kvpop {

// Ranking priority (score, or static priority under decay) of every token
// that becomes eligible in a prompt of n tokens, t in [S, max(S, n - W - D)),
// into out[u * cap + (t - S)].  The prefill scorer kernels, run over the whole
// prompt as one chunk.  Returns 0, -1 (CUDA) or -2 (more tokens than cap).
int launch_prompt_scores(const LayerArgs& a, int dtype, const void* k, const void* v, int n, const float* ext,
                         float* out, int cap, cudaStream_t st);

// Rows of query heads one fp32 attention CTA computes (query positions x G;
// the bf16 tensor-core kernel takes 256 rows).
constexpr int kPaRows = 64;
// Candidate keys staged per tile.
constexpr int kPaKeys = 32;
// Largest sort handled in shared memory (keys); larger sorts run in the workspace.
constexpr int kPaSmemSortKeys = 16384;
// Largest bitmap (32-bit words) kept in shared memory.
constexpr int kPaSmemBitmapWords = 4096;

struct PrefillAttnPlan {
  int n;            // prompt tokens
  int ne;           // tokens that become eligible in the prompt: max(0, n - W - D - S)
  int npow;         // sort length: next power of two >= max(ne, 1)
  int words;        // bitmap words: (ne + 31) / 32, at least 1
  int qt;           // query positions per attention CTA: 64 / G (fp32) or 256 / G (bf16)
  int cand_cap;     // candidate keys of one CTA at most: S + K + qt + W + D
  size_t cut_off, score_off, order_off, keys_off, bits_off, total;   // workspace layout (bytes)
  bool keys_global, bits_global;
};

// Plans the workspace and launch shapes; returns 0 or -2 (shape not supported).
int plan_prefill_attention(const LayerArgs& a, int dtype, int n, PrefillAttnPlan* p);

// Prompt scores, cutoffs, then attention, on `st` (reuse_cutoffs: the
// attention alone, from the cutoffs already in the workspace).  cut, scores,
// keys and bits point into the caller's workspace at the plan's offsets.
// Returns 0, -1 (CUDA) or -2.
int launch_prefill_attention(const LayerArgs& a, int dtype, const PrefillAttnPlan& p, const void* q, const void* k,
                             const void* v, const float* ext, void* out, float* lse, uint8_t* workspace,
                             cudaStream_t st, bool reuse_cutoffs = false);

// Whole-prompt cache build from the cutoffs of a launch_prefill_attention on
// the same workspace (the layer must be empty): the tokens kept to the end
// (cutoff "never") go to the long-range slots in ascending position order,
// with their ranking priorities.  Returns 0 or -1.
int launch_place_kept(const LayerArgs& a, int dtype, const PrefillAttnPlan& p, const void* k, const void* v,
                      const uint8_t* workspace, cudaStream_t st);

// The prompt's sinks, window and staging tokens to their slots (the prefill
// builder's write step for one whole-prompt chunk).  Returns 0 or -1.
int launch_prompt_write(const LayerArgs& a, int dtype, const void* k, const void* v, int n, const float* ext,
                        cudaStream_t st);

}  // namespace kvpop
