// The C ABI of liblvq: argument validation, layouts, and kernel launches.
#include <math.h>
#include <string.h>

#include <mutex>

#include "lvq_common.cuh"

using namespace lvq;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// LoopVQ shape rules ("LoopVQ summary", "how it differs": Tc divides T and G,
// one code covers c = G/Tc channels of each step; "premises and limits": 8-bit
// codes, K = 256, 8-token pages), then this build's kernel set.
lvq_status check_cfg(const lvq_config* c, bool need_table = true) {
  if (!c) return LVQ_EINVAL;
  if (c->n_layers < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->head_dim < 2 || c->T < 1 ||
      c->Tc < 1 || c->G < 1 || c->n_sink < 0 || c->n_recent < 0 || c->max_batch < 1 ||
      c->max_ctx < 1 || c->max_splits < 1 || !(c->rope_base > 0.f) || !isfinite(c->rope_base))
    return LVQ_EINVAL;
  if (c->T % c->Tc || c->G % c->Tc || c->n_q_heads % c->n_kv_heads || c->head_dim % 2)
    return LVQ_EINVAL;
  const int cc = c->G / c->Tc;
  if (c->head_dim % cc || (c->head_dim / cc) % 2) return LVQ_EINVAL;
  if (c->K != kEntries || c->page_tokens != kPage) return LVQ_EUNSUPPORTED;
  if (!decode_supported(c->head_dim, cc) || !encode_supported(c->G, cc)) return LVQ_EUNSUPPORTED;
  if (c->max_splits > 256 || c->max_ctx > (1 << 28)) return LVQ_EUNSUPPORTED;
  if (c->n_sink + c->n_recent + kPage > decode_bf16_capacity(c->head_dim, cc)) return LVQ_EUNSUPPORTED;
  // pool mode: a page table (16-byte aligned: the decode reads it in 16-byte pieces)
  if (c->pool_pages < 0 || c->reserved_ != 0) return LVQ_EINVAL;
  if (c->page_table && !aligned16(c->page_table)) return LVQ_EINVAL;
  if (c->pool_pages == 0 && c->page_table) return LVQ_EINVAL;
  if (need_table && c->pool_pages > 0 && !c->page_table) return LVQ_EINVAL;
  return LVQ_OK;
}

// test hook state (lvq_debug_faults); the defaults leave every kernel as in normal use
static long debug_wait_iters = kWaitIters;
static int debug_fault = 0;
// lvq_decode_max_ctas (0: one decode CTA per work item)
static int decode_max_ctas = 0;

Geo make_geo(const lvq_config* c) {
  Geo g;
  g.L = c->n_layers; g.H = c->n_kv_heads; g.Hq = c->n_q_heads; g.d = c->head_dim;
  g.T = c->T; g.Tc = c->Tc; g.G = c->G; g.c = c->G / c->Tc; g.ng = g.d / g.c; g.nblk = g.T / g.Tc;
  g.S = c->n_sink; g.W = c->n_recent; g.R = c->n_recent + kPage;
  const int max_coded = c->max_ctx > c->n_sink ? c->max_ctx - c->n_sink : 0;
  g.P = max_coded > 0 ? (max_coded + kPage - 1) / kPage : 1;
  g.B = c->max_batch; g.max_ctx = c->max_ctx; g.max_splits = c->max_splits;
  g.RC = max((c->max_ctx + kPage - 1) / kPage, 64) + 16;   // rows cover offsets up to 512 positions
  g.page_bytes = g.ng * kPage;
  g.wait_iters = debug_wait_iters;
  g.fault = debug_fault;
  g.max_ctas = decode_max_ctas;
  g.pool = c->pool_pages;
  g.pts = (g.P + 3) / 4 * 4;       // page-table row: whole 16-byte pieces
  g.pt = c->page_table;
  return g;
}

void fill_layout(const Geo& g, lvq_layout* o) {
  memset(o, 0, sizeof(*o));
  o->c = g.c; o->n_groups = g.ng; o->n_blocks = g.nblk; o->ring_tokens = g.R; o->max_pages = g.P;
  o->page_bytes = g.page_bytes; o->rope_coarse = g.RC;
  int64_t st = 1;
  if (g.pool == 0) {
    const int64_t idims[8] = {g.L, g.nblk, g.B, g.H, 2, g.P, g.ng, kPage};
    for (int i = 7; i >= 0; --i) { o->idx_strides[i] = st; st *= idims[i]; }
  } else {
    const int64_t idims[7] = {g.L, g.nblk, g.H, 2, g.pool, g.ng, kPage};
    for (int i = 6; i >= 0; --i) { o->idx_strides[i] = st; st *= idims[i]; }
    o->page_table_stride = g.pts;
    o->page_table_bytes = (size_t)g.B * g.pts * 4;
  }
  o->idx_bytes = (size_t)st;
  const int64_t cdims[7] = {g.L, 2, g.nblk, g.H, g.ng, kEntries, g.G};
  st = 1;
  for (int i = 6; i >= 0; --i) { o->cb_strides[i] = st; st *= cdims[i]; }
  o->cb_bytes = (size_t)st * 2;
  const int64_t pdims[8] = {g.L, 2, g.nblk, g.H, g.Tc, kEntries, g.ng, g.c};
  st = 1;
  for (int i = 7; i >= 0; --i) { o->cbp_strides[i] = st; st *= pdims[i]; }
  o->cbp_bytes = (size_t)st * 2;
  o->cb_norm_bytes = (size_t)g.L * 2 * g.nblk * g.H * g.ng * kEntries * 4;
  const int64_t sdims[7] = {g.L, 2, g.T, g.B, g.H, g.S, g.d};
  st = 1;
  for (int i = 6; i >= 0; --i) { o->sink_strides[i] = st; st *= sdims[i]; }
  o->sink_bytes = (size_t)st * 2;
  const int64_t rdims[7] = {g.L, 2, g.T, g.B, g.H, g.R, g.d};
  st = 1;
  for (int i = 6; i >= 0; --i) { o->ring_strides[i] = st; st *= rdims[i]; }
  o->ring_bytes = (size_t)st * 2;
  o->rope_bytes = (size_t)(g.RC + kPage) * (g.d / 2) * 2 * 4;
  o->workspace_bytes = ws_partial_floats(g) * 4 + (size_t)g.B * g.Hq * 4;
}

// Re-derives the layout and checks the caller's copy matches it.
lvq_status check_all(const lvq_config* cfg, const lvq_layout* lay, Geo* g) {
  lvq_status s = check_cfg(cfg);
  if (s != LVQ_OK) return s;
  if (!lay) return LVQ_EINVAL;
  *g = make_geo(cfg);
  lvq_layout ref;
  fill_layout(*g, &ref);
  if (memcmp(&ref, lay, sizeof(ref)) != 0) return LVQ_EINVAL;
  return LVQ_OK;
}

// The library runs on sm_100 devices only.
lvq_status check_device() {
  static int ok[kMaxDevices] = {};   // 0 unknown, 1 good, -1 bad
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LVQ_EDEVICE;
  if (dev < kMaxDevices && ok[dev] == 1) return LVQ_OK;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return LVQ_EDEVICE;
  const bool good = major == 10;
  if (dev < kMaxDevices) ok[dev] = good ? 1 : -1;
  return good ? LVQ_OK : LVQ_EDEVICE;
}

lvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LVQ_OK : LVQ_ECUDA; }

}  // namespace

extern "C" {

lvq_status lvq_cache_layout(const lvq_config* cfg, lvq_layout* out) {
  if (!out) return LVQ_EINVAL;
  lvq_status s = check_cfg(cfg, false);   // the layout does not depend on the page table's address
  if (s != LVQ_OK) return s;
  fill_layout(make_geo(cfg), out);
  return LVQ_OK;
}

const char* lvq_status_string(lvq_status s) {
  switch (s) {
    case LVQ_OK: return "ok";
    case LVQ_EINVAL: return "invalid argument";
    case LVQ_EUNSUPPORTED: return "shape not supported by this build";
    case LVQ_ECAPACITY: return "request exceeds the cache layout's capacity";
    case LVQ_ECUDA: return "CUDA call or kernel launch failed";
    case LVQ_ETIMEOUT: return "bounded device-side wait expired";
    case LVQ_EDEVICE: return "no usable sm_100 device";
  }
  return "unknown status";
}

lvq_status lvq_pack_codebooks(const lvq_config* cfg, const lvq_layout* lay, const void* cb, void* cbp,
                              float* cb_norm, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (!cb || !cbp || !aligned16(cb) || !aligned16(cbp) || (cb_norm && !aligned16(cb_norm)))
    return LVQ_EINVAL;
  if ((s = check_device()) != LVQ_OK) return s;
  return cuda_status(launch_pack(g, static_cast<const __nv_bfloat16*>(cb), static_cast<__nv_bfloat16*>(cbp),
                                 cb_norm, static_cast<cudaStream_t>(stream)));
}

lvq_status lvq_rope_table(const lvq_config* cfg, const lvq_layout* lay, float* rope, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (!rope || !aligned16(rope)) return LVQ_EINVAL;
  if ((s = check_device()) != LVQ_OK) return s;
  return cuda_status(launch_rope_table(g, cfg->rope_base, rope, static_cast<cudaStream_t>(stream)));
}

lvq_status lvq_encode_prefill(const lvq_config* cfg, const lvq_layout* lay, int32_t layer, int32_t req,
                              const void* kv, int64_t kv_tok_stride, int32_t kv_tokens, int32_t tok_begin,
                              int32_t n_tok, int32_t coded_offset, const void* cb, uint8_t* idx,
                              int32_t* dev_status, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (layer < -1 || layer >= g.L || req < 0 || req >= g.B || n_tok < 0 || tok_begin < 0 ||
      kv_tokens < 0 || (int64_t)tok_begin + n_tok > kv_tokens || coded_offset < 0 ||
      (int64_t)coded_offset + n_tok > (int64_t)g.P * kPage || kv_tok_stride < (int64_t)g.H * g.d)
    return LVQ_EINVAL;
  if (n_tok > 0 && (!kv || !cb || !idx || !aligned16(kv) || !aligned16(cb) || !aligned16(idx)))
    return LVQ_EINVAL;
  if ((s = check_device()) != LVQ_OK) return s;
  // tensor-core encoder where its tiles fit (c in {4, 8}, 16-byte token rows); the fp64
  // direct-form encoder otherwise.  Both return the exact nearest entry.
  if (encode_tc_supported(g.G, g.c) && kv_tok_stride % 8 == 0)
    return cuda_status(launch_encode_tc(g, layer, req, static_cast<const __nv_bfloat16*>(kv), kv_tok_stride,
                                        kv_tokens, tok_begin, n_tok, coded_offset,
                                        static_cast<const __nv_bfloat16*>(cb), idx, dev_status,
                                        static_cast<cudaStream_t>(stream)));
  return cuda_status(launch_encode_prefill(g, layer, req, static_cast<const __nv_bfloat16*>(kv), kv_tok_stride,
                                           kv_tokens, tok_begin, n_tok, coded_offset,
                                           static_cast<const __nv_bfloat16*>(cb), idx, dev_status,
                                           static_cast<cudaStream_t>(stream)));
}

lvq_status lvq_kmeans_update(const lvq_config* cfg, const lvq_layout* lay, int32_t layer, int32_t req,
                             const void* kv, int64_t kv_tok_stride, int32_t kv_tokens, int32_t tok_begin,
                             int32_t n_tok, int32_t coded_offset, const uint8_t* idx, void* cb, uint32_t* counts,
                             int32_t* dev_status, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (layer < 0 || layer >= g.L || req < 0 || req >= g.B || n_tok < 0 || tok_begin < 0 ||
      kv_tokens < 0 || (int64_t)tok_begin + n_tok > kv_tokens || coded_offset < 0 ||
      (int64_t)coded_offset + n_tok > (int64_t)g.P * kPage || kv_tok_stride < (int64_t)g.H * g.d)
    return LVQ_EINVAL;
  if (!kv || !cb || !idx || !aligned16(kv) || !aligned16(cb) || !aligned16(idx) ||
      (counts && !aligned16(counts)))
    return LVQ_EINVAL;
  if (g.ng % (64 / g.G) != 0 || kv_tok_stride % 8 != 0 || g.pool) return LVQ_EUNSUPPORTED;
  if ((s = check_device()) != LVQ_OK) return s;
  return cuda_status(launch_kmeans_update(g, layer, req, static_cast<const __nv_bfloat16*>(kv), kv_tok_stride,
                                          kv_tokens, tok_begin, n_tok, coded_offset, idx,
                                          static_cast<__nv_bfloat16*>(cb), counts, dev_status,
                                          static_cast<cudaStream_t>(stream)));
}

lvq_status lvq_encode_page(const lvq_config* cfg, const lvq_layout* lay, int32_t batch, const int32_t* ctx_len,
                           int32_t* coded_len, const void* ring, const void* cb, const float* cb_norm,
                           uint8_t* idx, int32_t* dev_status, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (batch < 0 || batch > g.B) return LVQ_EINVAL;
  if (batch > kPageMaxBatch) return LVQ_EUNSUPPORTED;
  if (batch > 0 && (!ctx_len || !coded_len || !ring || !cb || !cb_norm || !idx || !aligned16(ring) ||
                    !aligned16(cb) || !aligned16(cb_norm) || !aligned16(idx)))
    return LVQ_EINVAL;
  if ((s = check_device()) != LVQ_OK) return s;
  return cuda_status(launch_encode_page(g, batch, ctx_len, coded_len, static_cast<const __nv_bfloat16*>(ring),
                                        static_cast<const __nv_bfloat16*>(cb), cb_norm, idx, dev_status,
                                        static_cast<cudaStream_t>(stream)));
}

lvq_status lvq_decode_attention(const lvq_config* cfg, const lvq_layout* lay, int32_t layer, int32_t step,
                                int32_t batch, const void* q, const int32_t* ctx_len,
                                const int32_t* coded_len, const void* sink, const void* ring,
                                const uint8_t* idx, const void* cbp, const float* rope, int32_t num_splits,
                                float* workspace, float* out, float* lse, float* split_lse,
                                int32_t* dev_status, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (layer < 0 || layer >= g.L || step < 0 || step >= g.T || batch < 0 || batch > g.B || num_splits < 1 ||
      num_splits > g.max_splits)
    return LVQ_EINVAL;
  if (batch > 0) {
    const void* ptrs[] = {q, sink, ring, idx, cbp, rope, workspace, out, lse};
    for (const void* p : ptrs)
      if (!p || !aligned16(p)) return LVQ_EINVAL;
    if (!ctx_len || !coded_len || (split_lse && ((uintptr_t)split_lse & 3u))) return LVQ_EINVAL;
  }
  if ((s = check_device()) != LVQ_OK) return s;
  return cuda_status(launch_decode(g, layer, step, batch, static_cast<const __nv_bfloat16*>(q), ctx_len,
                                   coded_len, static_cast<const __nv_bfloat16*>(sink),
                                   static_cast<const __nv_bfloat16*>(ring), idx,
                                   static_cast<const __nv_bfloat16*>(cbp), rope, num_splits, workspace, out,
                                   lse, split_lse, dev_status, static_cast<cudaStream_t>(stream)));
}

lvq_status lvq_dequantize(const lvq_config* cfg, const lvq_layout* lay, int32_t layer, int32_t step,
                          int32_t req, int32_t kv, const uint8_t* idx, const void* cbp, int32_t tok_begin,
                          int32_t n_tok, void* out, void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (layer < 0 || layer >= g.L || step < 0 || step >= g.T || req < 0 || req >= g.B || (kv != 0 && kv != 1) ||
      tok_begin < 0 || n_tok < 0 || (int64_t)tok_begin + n_tok > (int64_t)g.P * kPage)
    return LVQ_EINVAL;
  if (n_tok > 0 && (!idx || !cbp || !out || !aligned16(idx) || !aligned16(cbp) || !aligned16(out)))
    return LVQ_EINVAL;
  if ((s = check_device()) != LVQ_OK) return s;
  return cuda_status(launch_dequantize(g, layer, step, req, kv, idx, static_cast<const __nv_bfloat16*>(cbp),
                                       tok_begin, n_tok, static_cast<__nv_bfloat16*>(out),
                                       static_cast<cudaStream_t>(stream)));
}


lvq_status lvq_debug_faults(int64_t wait_iters, int32_t fault_mask) {
  if (fault_mask & ~(kFaultDecodeDropChunk | kFaultKmeansDropTile)) return LVQ_EINVAL;
  debug_wait_iters = wait_iters > 0 ? (long)wait_iters : kWaitIters;
  debug_fault = fault_mask;
  return LVQ_OK;
}

lvq_status lvq_decode_max_ctas(int32_t max_ctas) {
  if (max_ctas < 0) return LVQ_EINVAL;
  decode_max_ctas = max_ctas;
  return LVQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------- allocation-free decode
//
// Some callers cannot allocate device memory for the decode workspace: for
// example a plugin running inside a serving engine whose memory pool owns the
// whole device, or a deployment that fixes its memory budget at start-up and
// forbids allocations afterwards.  For them lvq_decode_attention_noalloc uses
// a workspace that lives in the library itself: the file-scope device array
// below, which every GPU that loads the library holds until the process exits.

namespace {

constexpr size_t kNoallocWorkspaceBytes = size_t(4) << 20;   // the stated maximum: 4 MiB
static __device__ __align__(256) float g_noalloc_workspace[kNoallocWorkspaceBytes / sizeof(float)];

// Device address of g_noalloc_workspace for the current device and context.  In host code
// the array's name is only a stand-in, never a device address, so the address is looked up
// with cudaGetSymbolAddress with that device current: once per device, and again only if the
// device's current context changed since (after cudaDeviceReset the module is loaded anew and
// the array may move).  The lookup runs under a lock, so host threads that make their first
// calls at the same time do not race on the cache.
using PFN_ctx_get_current = CUresult (*)(CUcontext*);

CUcontext current_context() {
  static PFN_ctx_get_current fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_ctx_get_current>(p);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

float* noalloc_workspace(int dev) {
  static std::mutex mu;
  static CUcontext ctx[kMaxDevices] = {};
  static float* addr[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  const CUcontext cur = current_context();
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || ctx[dev] != cur) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<float*>(p);
    ctx[dev] = cur;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

lvq_status lvq_decode_attention_noalloc(const lvq_config* cfg, const lvq_layout* lay, int32_t layer, int32_t step,
                                        int32_t batch, const void* q, const int32_t* ctx_len,
                                        const int32_t* coded_len, const void* sink, const void* ring,
                                        const uint8_t* idx, const void* cbp, const float* rope, int32_t num_splits,
                                        float* out, float* lse, float* split_lse, int32_t* dev_status,
                                        void* stream) {
  Geo g;
  lvq_status s = check_all(cfg, lay, &g);
  if (s != LVQ_OK) return s;
  if (lay->workspace_bytes > kNoallocWorkspaceBytes) return LVQ_ECAPACITY;
  if (layer < 0 || layer >= g.L || step < 0 || step >= g.T || batch < 0 || batch > g.B || num_splits < 1 ||
      num_splits > g.max_splits)
    return LVQ_EINVAL;
  if (batch > 0) {
    const void* ptrs[] = {q, sink, ring, idx, cbp, rope, out, lse};
    for (const void* p : ptrs)
      if (!p || !aligned16(p)) return LVQ_EINVAL;
    if (!ctx_len || !coded_len || (split_lse && ((uintptr_t)split_lse & 3u))) return LVQ_EINVAL;
  }
  if ((s = check_device()) != LVQ_OK) return s;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LVQ_ECUDA;
  float* ws = noalloc_workspace(dev);
  if (!ws) return LVQ_ECUDA;
  if (batch == 0) return LVQ_OK;
  // the merge counters after the partials must start at zero (a previous call that
  // failed part-way could have left some set); the partials need no clearing
  const size_t partial_floats = ws_partial_floats(g);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws + partial_floats, 0, (size_t)g.B * g.Hq * sizeof(int32_t), st) != cudaSuccess)
    return LVQ_ECUDA;
  return cuda_status(launch_decode(g, layer, step, batch, static_cast<const __nv_bfloat16*>(q), ctx_len, coded_len,
                                   static_cast<const __nv_bfloat16*>(sink), static_cast<const __nv_bfloat16*>(ring),
                                   idx, static_cast<const __nv_bfloat16*>(cbp), rope, num_splits, ws, out, lse,
                                   split_lse, dev_status, st));
}

}  // extern "C"
