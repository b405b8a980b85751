// Host side of the KVpop C ABI (include/kvpop.h): validation, device buffer
// layout, host mirrors of the per-layer counters, kernel launches.
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/kvpop.h"
#include "kvpop_internal.cuh"
#include "kvpop_prefill_attn.cuh"

using namespace kvpop;

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Layout {
  int units, NS, G, esize, row_bytes, cap, kslots;
  size_t kv_off, kv_stride, pos_off, pos_stride, score_off, score_stride, state_off, state_stride;
  size_t layer_off, dec_off, dec_stride;
  size_t pacc_off, pml_off, ticket_off, pre_score_off, pre_tgt_off, err_off, total;
  size_t mlstm_off, mlstm_stride;   // mLSTM states per layer (0 bytes for the stateless scorers)
};

// The mLSTM scorer decides (not caller scores).
bool mlstm_active(const kvpop_config* c) {
  return c->scorer_kind == KVPOP_SCORER_MLSTM && !(c->flags & KVPOP_FLAG_EXTERNAL_SCORES);
}

bool hidden_supported(int h) { return h == 0 || h == 32 || h == 64 || h == 128; }   // 0: linear scorer

int validate(const kvpop_config* c) {
  if (!c) return KVPOP_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_layers < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1) return KVPOP_ERR_BAD_SHAPE;
  if (c->n_q_heads % c->n_kv_heads != 0) return KVPOP_ERR_BAD_SHAPE;
  if (c->dtype != KVPOP_DTYPE_F32 && c->dtype != KVPOP_DTYPE_BF16) return KVPOP_ERR_INVALID_ARG;
  if (c->sinks < 0 || c->window < 1 || c->topk < 0 || c->delay < 0) return KVPOP_ERR_BAD_SHAPE;
  if (c->max_context < 1 || c->max_prefill_chunk < 0) return KVPOP_ERR_BAD_SHAPE;
  if (c->log_decay != nullptr && c->max_context > (1 << 24)) return KVPOP_ERR_BAD_SHAPE;
  if ((c->flags & ~(KVPOP_FLAG_EXTERNAL_SCORES | KVPOP_FLAG_DEBUG_CHECKS)) != 0) return KVPOP_ERR_INVALID_ARG;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (!decode_supported(c->dtype, c->head_dim, G)) return KVPOP_ERR_BAD_SHAPE;
  if (c->scorer_kind != KVPOP_SCORER_MLP && c->scorer_kind != KVPOP_SCORER_MLSTM) return KVPOP_ERR_INVALID_ARG;
  if (c->scorer_kind == KVPOP_SCORER_MLSTM) {
    if (c->mlstm_p < 1 || c->mlstm_p > 16 || c->mlstm_dv < 1 || c->mlstm_dv > 32) return KVPOP_ERR_BAD_SHAPE;
    if (c->head_dim != 64 && c->head_dim != 128) return KVPOP_ERR_BAD_SHAPE;
    if (mlstm_active(c) && (!c->mlstm_w || (reinterpret_cast<uintptr_t>(c->mlstm_w) & 15u) != 0))
      return KVPOP_ERR_INVALID_ARG;
  } else if (!(c->flags & KVPOP_FLAG_EXTERNAL_SCORES)) {
    if (!hidden_supported(c->scorer_hidden)) return KVPOP_ERR_BAD_SHAPE;
    if (!c->w1 || !c->b2 || (c->scorer_hidden > 0 && (!c->b1 || !c->w2))) return KVPOP_ERR_INVALID_ARG;
  }
  const double budget = static_cast<double>(c->sinks) + c->window + c->topk;
  if (budget + c->delay > 2147483647.0 / 2) return KVPOP_ERR_BAD_SHAPE;
  if (c->ref_context > 0) {
    if (!(c->compression_ratio >= 0.f && c->compression_ratio < 1.f)) return KVPOP_ERR_INVALID_ARG;
    if (std::fabs((1.0 - c->compression_ratio) * c->ref_context - budget) > 0.5) return KVPOP_ERR_INVALID_ARG;
  }
  return KVPOP_OK;
}

Layout make_layout(const kvpop_config* c) {
  Layout L{};
  L.units = c->batch * c->n_kv_heads;
  L.NS = c->sinks + c->window + c->delay + c->topk;
  L.G = c->n_q_heads / c->n_kv_heads;
  L.esize = c->dtype == KVPOP_DTYPE_F32 ? 4 : 2;
  L.row_bytes = 2 * c->head_dim * L.esize;
  L.cap = c->max_prefill_chunk > 0 ? c->max_prefill_chunk : 1;
  L.kslots = c->topk > 0 ? c->topk : 1;
  const size_t units = L.units, NS = L.NS, layers = c->n_layers;
  size_t off = 0;
  L.kv_stride = align256(units * NS * L.row_bytes);
  L.kv_off = off; off += layers * L.kv_stride;
  L.pos_stride = align256(units * NS * 4);
  L.pos_off = off; off += layers * L.pos_stride;
  L.score_stride = align256(units * NS * 4);
  L.score_off = off; off += layers * L.score_stride;
  L.state_stride = align256(units * 16);
  L.state_off = off; off += layers * L.state_stride;
  // after state_off: zeroed at creation (an mLSTM state starts at C = 0, n = 0, m = 0)
  L.mlstm_stride = c->scorer_kind == KVPOP_SCORER_MLSTM
                       ? align256(units * static_cast<size_t>(mlstm_state_doubles(c->mlstm_p, c->mlstm_dv)) * 8)
                       : 0;
  L.mlstm_off = off; off += layers * L.mlstm_stride;
  L.layer_off = off; off += align256(layers * sizeof(LayerState));
  L.dec_stride = align256(2 * units * sizeof(Decision));
  L.dec_off = off; off += layers * L.dec_stride;
  L.pacc_off = off; off += align256(units * kMaxSeg * L.G * c->head_dim * 4);
  L.pml_off = off; off += align256(units * kMaxSeg * L.G * 2 * 4);
  L.ticket_off = off; off += align256(units * 4);
  L.pre_score_off = off; off += align256(units * static_cast<size_t>(L.cap) * 4);
  L.pre_tgt_off = off; off += align256(units * static_cast<size_t>(L.kslots) * 4);
  L.err_off = off; off += 256;
  L.total = off;
  return L;
}

}  // namespace

struct kvpop_handle {
  kvpop_config cfg;
  Layout lay;
  uint8_t* mem;
  int device;
  int num_sms;
  std::vector<int> n_seen;   // host mirror of each layer's position counter
  std::vector<int> n_topk;   // host mirror of each layer's long-range fill
  std::vector<char> decoding;
  std::vector<CUtensorMap> maps;  // per layer: TMA view of the cache rows
  int test_hook = 0;              // failure injection (KVPOP_TEST_HOOKS builds only)
};

namespace {

LayerArgs layer_args(const kvpop_handle* h, int layer) {
  const kvpop_config& c = h->cfg;
  const Layout& L = h->lay;
  LayerArgs a{};
  a.kv = h->mem + L.kv_off + layer * L.kv_stride;
  a.pos = reinterpret_cast<int32_t*>(h->mem + L.pos_off + layer * L.pos_stride);
  a.score = reinterpret_cast<float*>(h->mem + L.score_off + layer * L.score_stride);
  a.state = reinterpret_cast<int32_t*>(h->mem + L.state_off + layer * L.state_stride);
  a.layer = reinterpret_cast<LayerState*>(h->mem + L.layer_off) + layer;
  a.dec = reinterpret_cast<Decision*>(h->mem + L.dec_off + layer * L.dec_stride);
  const size_t hid = c.scorer_hidden, d2 = 2 * static_cast<size_t>(c.head_dim), H = c.n_kv_heads;
  if (c.w1) {
    a.w1 = c.w1 + layer * H * (hid > 0 ? hid : 1) * d2;   // linear scorer: one row per head
    a.b1 = (hid > 0 && c.b1) ? c.b1 + layer * H * hid : nullptr;
    a.w2 = (hid > 0 && c.w2) ? c.w2 + layer * H * hid : nullptr;
    a.b2 = c.b2 + layer * H;
  }
  a.err = reinterpret_cast<int32_t*>(h->mem + L.err_off);
  a.units = L.units;
  a.Hkv = c.n_kv_heads;
  a.Hq = c.n_q_heads;
  a.G = L.G;
  a.d = c.head_dim;
  a.S = c.sinks;
  a.W = c.window;
  a.D = c.delay;
  a.K = c.topk;
  a.NS = L.NS;
  a.hidden = c.scorer_hidden;
  a.max_context = c.max_context;
  a.flags = c.flags;
  a.row_bytes = L.row_bytes;
  a.log_decay = c.log_decay ? c.log_decay + static_cast<size_t>(layer) * H : nullptr;
  a.test_hook = h->test_hook;
  a.mlstm = mlstm_active(&c) ? 1 : 0;
  if (c.scorer_kind == KVPOP_SCORER_MLSTM) {
    a.mp = c.mlstm_p;
    a.mdv = c.mlstm_dv;
    a.mw = c.mlstm_w ? c.mlstm_w + static_cast<size_t>(layer) * H * mlstm_head_floats(c.mlstm_p, c.mlstm_dv, c.head_dim)
                     : nullptr;
    a.mstate = reinterpret_cast<double*>(h->mem + L.mlstm_off + layer * L.mlstm_stride);
  }
  return a;
}

DecodeScratch decode_scratch(const kvpop_handle* h) {
  DecodeScratch s;
  s.part_acc = reinterpret_cast<float*>(h->mem + h->lay.pacc_off);
  s.part_ml = reinterpret_cast<float*>(h->mem + h->lay.pml_off);
  s.ticket = reinterpret_cast<int32_t*>(h->mem + h->lay.ticket_off);
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool on_device(const void* p) {
  if (!p) return false;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

__global__ void poison_kernel(int32_t* err, int32_t bits) { atomicOr(err, bits); }

}  // namespace

extern "C" {

int kvpop_cache_bytes(const kvpop_config* cfg, size_t* bytes) {
  if (!bytes) return KVPOP_ERR_INVALID_ARG;
  const int v = validate(cfg);
  if (v != KVPOP_OK) return v;
  *bytes = make_layout(cfg).total;
  return KVPOP_OK;
}

int kvpop_create(const kvpop_config* cfg, void* dev_mem, size_t bytes, kvpop_handle** out) {
  if (!out) return KVPOP_ERR_INVALID_ARG;
  *out = nullptr;
  const int v = validate(cfg);
  if (v != KVPOP_OK) return v;
  const Layout L = make_layout(cfg);
  if (!dev_mem || bytes < L.total || (reinterpret_cast<uintptr_t>(dev_mem) & 255u) != 0)
    return KVPOP_ERR_INVALID_ARG;
  if (!on_device(dev_mem)) return KVPOP_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVPOP_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return KVPOP_ERR_CUDA;
  kvpop_handle* h = new (std::nothrow) kvpop_handle();
  if (!h) return KVPOP_ERR_INVALID_ARG;
  h->cfg = *cfg;
  h->lay = L;
  h->mem = static_cast<uint8_t*>(dev_mem);
  h->device = dev;
  h->num_sms = sms;
  h->n_seen.assign(cfg->n_layers, 0);
  h->n_topk.assign(cfg->n_layers, 0);
  h->decoding.assign(cfg->n_layers, 0);
  h->maps.resize(cfg->n_layers);
  for (int l = 0; l < cfg->n_layers; ++l) {
    if (make_decode_tensor_map(&h->maps[l], h->mem + L.kv_off + l * L.kv_stride, cfg->dtype, cfg->head_dim,
                               static_cast<int64_t>(L.units) * L.NS, L.row_bytes) != 0) {
      delete h;
      return KVPOP_ERR_CUDA;
    }
  }
  uint8_t* m = h->mem;
  bool ok = cudaMemset(m + L.kv_off, 0, cfg->n_layers * L.kv_stride) == cudaSuccess &&
            cudaMemset(m + L.pos_off, 0xff, cfg->n_layers * L.pos_stride) == cudaSuccess &&
            cudaMemset(m + L.score_off, 0, cfg->n_layers * L.score_stride) == cudaSuccess &&
            cudaMemset(m + L.state_off, 0, L.total - L.state_off) == cudaSuccess;
  for (int l = 0; ok && l < cfg->n_layers; ++l)
    ok = launch_decide(layer_args(h, l), cfg->dtype, 0, 0, nullptr) == 0;
  ok = ok && cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    delete h;
    return KVPOP_ERR_CUDA;
  }
  *out = h;
  return KVPOP_OK;
}

int kvpop_prefill(kvpop_handle* h, int32_t layer, const void* k, const void* v, int32_t n_tokens,
                  const float* ext_scores, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers || n_tokens < 0) return KVPOP_ERR_INVALID_ARG;
  if (n_tokens > h->cfg.max_prefill_chunk) return KVPOP_ERR_BAD_SHAPE;
  if (h->decoding[layer]) return KVPOP_ERR_ORDER;
  const bool ext = (h->cfg.flags & KVPOP_FLAG_EXTERNAL_SCORES) != 0;
  if (n_tokens > 0 && (!k || !v)) return KVPOP_ERR_INVALID_ARG;
  if (n_tokens > 0 && ext && !ext_scores) return KVPOP_ERR_INVALID_ARG;
  if (static_cast<int64_t>(h->n_seen[layer]) + n_tokens > h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  if (n_tokens == 0) return KVPOP_OK;
  const LayerArgs a = layer_args(h, layer);
  PrefillScratch ps;
  ps.new_score = reinterpret_cast<float*>(h->mem + h->lay.pre_score_off);
  ps.tgt = reinterpret_cast<int32_t*>(h->mem + h->lay.pre_tgt_off);
  ps.cap = h->lay.cap;
  const int n0 = h->n_seen[layer], c0 = h->n_topk[layer];
  const int r = launch_prefill(a, h->cfg.dtype, ps, k, v, n_tokens, n0, c0, ext ? ext_scores : nullptr,
                               static_cast<cudaStream_t>(stream));
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  if (r != 0) return KVPOP_ERR_CUDA;
  const int S = h->cfg.sinks, W = h->cfg.window, D = h->cfg.delay;
  const int e0 = std::max(S, n0 - W - D), e1 = std::max(S, n0 + n_tokens - W - D);
  const int n1 = n0 + n_tokens, c1 = std::min(h->cfg.topk, c0 + (e1 - e0));
  if (launch_decide(a, h->cfg.dtype, n1, c1, static_cast<cudaStream_t>(stream)) != 0) return KVPOP_ERR_CUDA;
  h->n_seen[layer] = n1;
  h->n_topk[layer] = c1;
  return KVPOP_OK;
}

namespace {
void advance_mirror(kvpop_handle* h, int layer) {
  const int S = h->cfg.sinks, W = h->cfg.window, D = h->cfg.delay;
  const int p = h->n_seen[layer];
  if (p - W - D >= S && h->n_topk[layer] < h->cfg.topk) h->n_topk[layer] += 1;
  h->n_seen[layer] = p + 1;
  h->decoding[layer] = 1;
}
}  // namespace

int kvpop_decode_append(kvpop_handle* h, int32_t layer, const void* k_new, const void* v_new,
                        const float* ext_score, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers) return KVPOP_ERR_INVALID_ARG;
  if (!k_new || !v_new) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return KVPOP_ERR_INVALID_ARG;
  const bool ext = (h->cfg.flags & KVPOP_FLAG_EXTERNAL_SCORES) != 0;
  if (ext && !ext_score) return KVPOP_ERR_INVALID_ARG;
  if (h->n_seen[layer] >= h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  const LayerArgs a = layer_args(h, layer);
  if (a.mlstm && launch_mlstm_step(a, h->cfg.dtype, k_new, v_new, static_cast<cudaStream_t>(stream)) != 0)
    return KVPOP_ERR_CUDA;
  if (launch_append(a, h->cfg.dtype, k_new, v_new, ext ? ext_score : nullptr, static_cast<cudaStream_t>(stream)) != 0)
    return KVPOP_ERR_CUDA;
  advance_mirror(h, layer);
  return KVPOP_OK;
}

int kvpop_decode_attend(kvpop_handle* h, int32_t layer, const void* q, void* out, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers) return KVPOP_ERR_INVALID_ARG;
  if (!q || !out) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out)) return KVPOP_ERR_INVALID_ARG;
  if (h->n_seen[layer] == 0) return KVPOP_ERR_ORDER;
  const LayerArgs a = layer_args(h, layer);
  const int r = launch_decode(h->maps[layer], a, h->cfg.dtype, decode_scratch(h), MODE_ATTEND, q, nullptr, nullptr,
                              nullptr, out, h->num_sms, static_cast<cudaStream_t>(stream));
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  return r == 0 ? KVPOP_OK : KVPOP_ERR_CUDA;
}

int kvpop_decode_step(kvpop_handle* h, int32_t layer, const void* q, const void* k_new, const void* v_new,
                      void* out, const float* ext_score, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers) return KVPOP_ERR_INVALID_ARG;
  if (!q || !out || !k_new || !v_new) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_new) || !aligned16(v_new)) return KVPOP_ERR_INVALID_ARG;
  const bool ext = (h->cfg.flags & KVPOP_FLAG_EXTERNAL_SCORES) != 0;
  if (ext && !ext_score) return KVPOP_ERR_INVALID_ARG;
  if (h->n_seen[layer] >= h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  const LayerArgs a = layer_args(h, layer);
  if (a.mlstm && launch_mlstm_step(a, h->cfg.dtype, k_new, v_new, static_cast<cudaStream_t>(stream)) != 0)
    return KVPOP_ERR_CUDA;
  const int r = launch_decode(h->maps[layer], a, h->cfg.dtype, decode_scratch(h), a.mlstm ? MODE_STEP_NODECIDE : MODE_STEP,
                              q, k_new, v_new, ext ? ext_score : nullptr, out, h->num_sms,
                              static_cast<cudaStream_t>(stream));
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  if (r != 0) return KVPOP_ERR_CUDA;
  advance_mirror(h, layer);
  return KVPOP_OK;
}

int kvpop_inspect(kvpop_handle* h, int32_t layer, int32_t* pos_out, float* score_out, int32_t* state_out,
                  void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers) return KVPOP_ERR_INVALID_ARG;
  const Layout& L = h->lay;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t n = static_cast<size_t>(L.units) * L.NS;
  if (pos_out && cudaMemcpyAsync(pos_out, h->mem + L.pos_off + layer * L.pos_stride, n * 4,
                                 cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KVPOP_ERR_CUDA;
  if (score_out && cudaMemcpyAsync(score_out, h->mem + L.score_off + layer * L.score_stride, n * 4,
                                   cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KVPOP_ERR_CUDA;
  if (state_out && cudaMemcpyAsync(state_out, h->mem + L.state_off + layer * L.state_stride,
                                   static_cast<size_t>(L.units) * 16, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KVPOP_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? KVPOP_OK : KVPOP_ERR_CUDA;
}

int kvpop_get_layout(const kvpop_handle* h, kvpop_layout_info* o) {
  if (!h || !o) return KVPOP_ERR_INVALID_ARG;
  const Layout& L = h->lay;
  o->kv_offset = L.kv_off; o->kv_layer_stride = L.kv_stride;
  o->pos_offset = L.pos_off; o->pos_layer_stride = L.pos_stride;
  o->score_offset = L.score_off; o->score_layer_stride = L.score_stride;
  o->state_offset = L.state_off; o->state_layer_stride = L.state_stride;
  o->slots_per_unit = L.NS;
  o->units = L.units;
  o->row_bytes = L.row_bytes;
  o->topk_base = h->cfg.sinks + h->cfg.window + h->cfg.delay;
  return KVPOP_OK;
}

int kvpop_get_error(kvpop_handle* h, int32_t* device_bits) {
  if (!h) return KVPOP_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return KVPOP_ERR_CUDA;
  int32_t bits = 0;
  if (cudaMemcpy(&bits, h->mem + h->lay.err_off, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return KVPOP_ERR_CUDA;
  if (device_bits) *device_bits = bits;
  if (bits == 0) return KVPOP_OK;
  if (bits & DEVERR_TIMEOUT) return KVPOP_ERR_TIMEOUT;
  if (bits == DEVERR_CONTEXT_OVERFLOW) return KVPOP_ERR_CONTEXT_OVERFLOW;
  return KVPOP_ERR_DEVICE;
}

int kvpop_clear_error(kvpop_handle* h, void* stream) {
  if (!h) return KVPOP_ERR_INVALID_ARG;
  return cudaMemsetAsync(h->mem + h->lay.err_off, 0, 4, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KVPOP_OK
             : KVPOP_ERR_CUDA;
}

int kvpop_debug_poison_error(kvpop_handle* h, int32_t bits, void* stream) {
  if (!h) return KVPOP_ERR_INVALID_ARG;
  poison_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<int32_t*>(h->mem + h->lay.err_off),
                                                                bits);
  return cudaGetLastError() == cudaSuccess ? KVPOP_OK : KVPOP_ERR_CUDA;
}

int kvpop_prefill_attention_workspace_bytes(const kvpop_handle* h, int32_t n_tokens, size_t* bytes) {
  if (!h || !bytes || n_tokens < 0) return KVPOP_ERR_INVALID_ARG;
  if (n_tokens > h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  PrefillAttnPlan p;
  if (plan_prefill_attention(layer_args(h, 0), h->cfg.dtype, n_tokens, &p) != 0) return KVPOP_ERR_BAD_SHAPE;
  *bytes = p.total;
  return KVPOP_OK;
}

int kvpop_prefill_attention(kvpop_handle* h, int32_t layer, const void* q, const void* k, const void* v,
                            int32_t n_tokens, const float* ext_scores, void* out, float* lse, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers || n_tokens < 0) return KVPOP_ERR_INVALID_ARG;
  if (n_tokens > h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  if (n_tokens == 0) return KVPOP_OK;
  if (!q || !k || !v || !out || !workspace) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return KVPOP_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return KVPOP_ERR_INVALID_ARG;
  const bool ext = (h->cfg.flags & KVPOP_FLAG_EXTERNAL_SCORES) != 0;
  if (ext && !ext_scores) return KVPOP_ERR_INVALID_ARG;
  const LayerArgs a = layer_args(h, layer);
  PrefillAttnPlan p;
  if (plan_prefill_attention(a, h->cfg.dtype, n_tokens, &p) != 0 || a.units > 65535) return KVPOP_ERR_BAD_SHAPE;
  if (workspace_bytes < p.total) return KVPOP_ERR_INVALID_ARG;
  const int r = launch_prefill_attention(a, h->cfg.dtype, p, q, k, v, ext ? ext_scores : nullptr, out, lse,
                                         static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  return r == 0 ? KVPOP_OK : KVPOP_ERR_CUDA;
}

int kvpop_prefill_attention_from_cutoffs(kvpop_handle* h, int32_t layer, const void* q, const void* k, const void* v,
                                         int32_t n_tokens, void* out, float* lse, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers || n_tokens < 0) return KVPOP_ERR_INVALID_ARG;
  if (n_tokens > h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  if (n_tokens == 0) return KVPOP_OK;
  if (!q || !k || !v || !out || !workspace) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return KVPOP_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return KVPOP_ERR_INVALID_ARG;
  const LayerArgs a = layer_args(h, layer);
  PrefillAttnPlan p;
  if (plan_prefill_attention(a, h->cfg.dtype, n_tokens, &p) != 0 || a.units > 65535) return KVPOP_ERR_BAD_SHAPE;
  if (workspace_bytes < p.total) return KVPOP_ERR_INVALID_ARG;
  const int r = launch_prefill_attention(a, h->cfg.dtype, p, q, k, v, nullptr, out, lse,
                                         static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream),
                                         true);
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  return r == 0 ? KVPOP_OK : KVPOP_ERR_CUDA;
}

int kvpop_prefill_with_attention(kvpop_handle* h, int32_t layer, const void* q, const void* k, const void* v,
                                 int32_t n_tokens, const float* ext_scores, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers || n_tokens < 0) return KVPOP_ERR_INVALID_ARG;
  if (h->decoding[layer] || h->n_seen[layer] != 0) return KVPOP_ERR_ORDER;
  if (n_tokens > h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  if (n_tokens == 0) return KVPOP_OK;
  if (!q || !k || !v || !out || !workspace) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return KVPOP_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return KVPOP_ERR_INVALID_ARG;
  const bool ext = (h->cfg.flags & KVPOP_FLAG_EXTERNAL_SCORES) != 0;
  if (ext && !ext_scores) return KVPOP_ERR_INVALID_ARG;
  const LayerArgs a = layer_args(h, layer);
  PrefillAttnPlan p;
  if (plan_prefill_attention(a, h->cfg.dtype, n_tokens, &p) != 0 || a.units > 65535) return KVPOP_ERR_BAD_SHAPE;
  if (workspace_bytes < p.total) return KVPOP_ERR_INVALID_ARG;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float* es = ext ? ext_scores : nullptr;
  int r = launch_prefill_attention(a, h->cfg.dtype, p, q, k, v, es, out, lse, ws, st);
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  if (r != 0) return KVPOP_ERR_CUDA;
  if (launch_place_kept(a, h->cfg.dtype, p, k, v, ws, st) != 0) return KVPOP_ERR_CUDA;
  if (launch_prompt_write(a, h->cfg.dtype, k, v, n_tokens, es, st) != 0) return KVPOP_ERR_CUDA;
  const int c1 = std::min(h->cfg.topk, p.ne);
  if (launch_decide(a, h->cfg.dtype, n_tokens, c1, st) != 0) return KVPOP_ERR_CUDA;
  h->n_seen[layer] = n_tokens;
  h->n_topk[layer] = c1;
  return KVPOP_OK;
}

int kvpop_debug_set_hook(kvpop_handle* h, int32_t hook) {
#ifdef KVPOP_TEST_HOOKS
  if (!h || hook < 0 || hook > TEST_HOOK_WITHHOLD_DONE) return KVPOP_ERR_INVALID_ARG;
  h->test_hook = hook;
  return KVPOP_OK;
#else
  (void)h;
  (void)hook;
  return KVPOP_ERR_INVALID_ARG;   // not a test build: no hook exists
#endif
}

int kvpop_destroy(kvpop_handle* h) {
  if (!h) return KVPOP_ERR_INVALID_ARG;
  delete h;
  return KVPOP_OK;
}

const char* kvpop_status_string(int s) {
  switch (s) {
    case KVPOP_OK: return "ok";
    case KVPOP_ERR_INVALID_ARG: return "invalid argument";
    case KVPOP_ERR_BAD_SHAPE: return "unsupported or inconsistent shape";
    case KVPOP_ERR_ORDER: return "call out of order";
    case KVPOP_ERR_CONTEXT_OVERFLOW: return "context overflow";
    case KVPOP_ERR_CUDA: return "CUDA runtime error";
    case KVPOP_ERR_DEVICE: return "device-side error recorded";
    case KVPOP_ERR_TIMEOUT: return "device-side wait timed out";
    case KVPOP_ERR_SCRATCH_LIMIT: return "problem needs more split-K scratch than the 16 MiB static buffer holds";
    default: return "unknown status";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// kvpop_decode_step_noalloc: the decode step with its split-K scratch in a
// static device buffer, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------

// Split-K partials [units][kMaxSeg][G][d] and [units][kMaxSeg][G][2] (fp32)
// and arrival tickets [units] (int32) of kvpop_decode_step_noalloc.  One copy
// per GPU, part of the module image; host code must not hand this name to a
// kernel (on the host it only stands for the symbol): the device address
// comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[KVPOP_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
uint8_t* g_noalloc_base[kNoallocMaxDevices];   // device address per device, looked up once

// Device address of g_noalloc_scratch on `dev`, which must be current.  The
// first call per device does the lookup (this is the set-up step that must
// happen before any stream capture).
int noalloc_base(int dev, uint8_t** base) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_base[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return KVPOP_ERR_CUDA;
    }
    g_noalloc_base[dev] = static_cast<uint8_t*>(p);
  }
  *base = g_noalloc_base[dev];
  return KVPOP_OK;
}

}  // namespace

extern "C" int kvpop_decode_step_noalloc(kvpop_handle* h, int32_t layer, const void* q, const void* k_new,
                                         const void* v_new, void* out, const float* ext_score, void* stream) {
  if (!h || layer < 0 || layer >= h->cfg.n_layers) return KVPOP_ERR_INVALID_ARG;
  if (!q || !out || !k_new || !v_new) return KVPOP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_new) || !aligned16(v_new)) return KVPOP_ERR_INVALID_ARG;
  const bool ext = (h->cfg.flags & KVPOP_FLAG_EXTERNAL_SCORES) != 0;
  if (ext && !ext_score) return KVPOP_ERR_INVALID_ARG;
  if (h->n_seen[layer] >= h->cfg.max_context) return KVPOP_ERR_CONTEXT_OVERFLOW;
  // the same split-K layout as the handle's own region, packed from offset 0
  const size_t units = h->lay.units, G = h->lay.G, d = h->cfg.head_dim;
  const size_t acc_bytes = align256(units * kMaxSeg * G * d * 4);
  const size_t ml_bytes = align256(units * kMaxSeg * G * 2 * 4);
  const size_t ticket_bytes = units * 4;
  if (acc_bytes + ml_bytes + align256(ticket_bytes) > KVPOP_NOALLOC_SCRATCH_BYTES) return KVPOP_ERR_SCRATCH_LIMIT;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVPOP_ERR_CUDA;
  if (dev != h->device || dev < 0 || dev >= kNoallocMaxDevices) return KVPOP_ERR_INVALID_ARG;
  uint8_t* base = nullptr;
  const int rb = noalloc_base(dev, &base);
  if (rb != KVPOP_OK) return rb;
  DecodeScratch sc;
  sc.part_acc = reinterpret_cast<float*>(base);
  sc.part_ml = reinterpret_cast<float*>(base + acc_bytes);
  sc.ticket = reinterpret_cast<int32_t*>(base + acc_bytes + ml_bytes);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the tickets count arrivals from zero; a call that gave up on a wait can
  // leave them non-zero, and another handle may have used more units
  if (cudaMemsetAsync(sc.ticket, 0, ticket_bytes, st) != cudaSuccess) return KVPOP_ERR_CUDA;
  const LayerArgs a = layer_args(h, layer);
  if (a.mlstm && launch_mlstm_step(a, h->cfg.dtype, k_new, v_new, st) != 0) return KVPOP_ERR_CUDA;
  const int r = launch_decode(h->maps[layer], a, h->cfg.dtype, sc, a.mlstm ? MODE_STEP_NODECIDE : MODE_STEP, q, k_new,
                              v_new, ext ? ext_score : nullptr, out, h->num_sms, st);
  if (r == -2) return KVPOP_ERR_BAD_SHAPE;
  if (r != 0) return KVPOP_ERR_CUDA;
  advance_mirror(h, layer);
  return KVPOP_OK;
}
