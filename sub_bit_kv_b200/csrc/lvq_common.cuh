// Internal definitions shared by liblvq's translation units (not installed).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lvq.h"

namespace lvq {

constexpr int kEntries = 256;   // 8-bit codes
constexpr int kPage = 8;        // tokens per page

// Geometry of one configuration, passed by value to every kernel.
struct Geo {
  int L, H, Hq, d, T, Tc, G, c, ng, nblk;
  int S, W, R, P, B, max_ctx, max_splits, RC;
  int page_bytes;
  long wait_iters;   // bound of every device-side wait (kWaitIters unless a test lowers it)
  int fault;         // test hook: kFault* bits, 0 in normal use
  int pool;          // pool mode: physical pages per (layer, block, head, K/V); 0: per-request streams
  int pts;           // page-table entries per request (pool mode)
  const int32_t* pt; // device page table [B][pts] (pool mode)
  int max_ctas;      // decode: CTA cap (lvq_decode_max_ctas; 0: one CTA per work item)
};
// Test hook bits (lvq_debug_faults): a copy that is never issued, so that a bounded wait
// runs out and the kernel reports LVQ_ETIMEOUT.
constexpr int kFaultDecodeDropChunk = 1;   // decode: the first code chunk of every CTA
constexpr int kFaultKmeansDropTile = 2;    // k-means update: the first tile of every CTA

// byte offset of the code stream [page][n_g][8] of (layer, blk, b, h, kv)
__host__ __device__ inline size_t idx_stream_off(const Geo& g, int layer, int blk, int b, int h, int kv) {
  return (((((size_t)layer * g.nblk + blk) * g.B + b) * g.H + h) * 2 + kv) * (size_t)g.P * g.page_bytes;
}
// Pool mode: byte offset of physical page 0 of the (layer, blk, h, kv) pool
__host__ __device__ inline size_t idx_pool_off(const Geo& g, int layer, int blk, int h, int kv) {
  return ((((size_t)layer * g.nblk + blk) * g.H + h) * 2 + kv) * (size_t)g.pool * g.page_bytes;
}
// Physical page of request b's logical page pg: itself outside pool mode, else the page
// table's entry; -1 if the entry is out of range (the caller reports LVQ_ECAPACITY)
__device__ inline int phys_page(const Geo& g, int b, int pg) {
  if (g.pool == 0) return pg;
  const int id = __ldg(g.pt + (size_t)b * g.pts + pg);
  return id >= 0 && id < g.pool ? id : -1;
}
// byte offset of physical page `phys` of the code stream of (layer, blk, b, h, kv)
__host__ __device__ inline size_t idx_page_off(const Geo& g, int layer, int blk, int b, int h, int kv, int phys) {
  return g.pool ? idx_pool_off(g, layer, blk, h, kv) + (size_t)phys * g.page_bytes
                : idx_stream_off(g, layer, blk, b, h, kv) + (size_t)phys * g.page_bytes;
}
// byte offset of group grp's code of coded token n (logical page n/8 is physical page phys)
__host__ __device__ inline size_t idx_code_off(const Geo& g, int layer, int blk, int b, int h, int kv, int phys,
                                               int n, int grp) {
  return idx_page_off(g, layer, blk, b, h, kv, phys) + grp * kPage + (n & 7);
}
// element offset of the packed step slice [256][ng][c] of (layer, kv, blk, h, s)
__host__ __device__ inline size_t cbp_slice_off(const Geo& g, int layer, int kv, int blk, int h, int s) {
  return (((((size_t)layer * 2 + kv) * g.nblk + blk) * g.H + h) * g.Tc + s) * (size_t)kEntries * g.d;
}
// element offset of the logical codebook [256][G] of (layer, kv, blk, h, grp)
__host__ __device__ inline size_t cb_off(const Geo& g, int layer, int kv, int blk, int h, int grp) {
  return (((((size_t)layer * 2 + kv) * g.nblk + blk) * g.H + h) * g.ng + grp) * (size_t)kEntries * g.G;
}
// element offset of token `i` of the sink of (layer, kv, step, b, h)
__host__ __device__ inline size_t sink_off(const Geo& g, int layer, int kv, int t, int b, int h, int i) {
  return ((((((size_t)layer * 2 + kv) * g.T + t) * g.B + b) * g.H + h) * g.S + i) * (size_t)g.d;
}
// element offset of ring slot `slot` of (layer, kv, step, b, h)
__host__ __device__ inline size_t ring_off(const Geo& g, int layer, int kv, int t, int b, int h, int slot) {
  return ((((((size_t)layer * 2 + kv) * g.T + t) * g.B + b) * g.H + h) * g.R + slot) * (size_t)g.d;
}

// fp32 partials of the decode workspace: [B][Hq][max_splits][coded, bf16][d + 2];
// the int32 merge counters [B][Hq] follow them.
__host__ __device__ inline size_t ws_partial_floats(const Geo& g) {
  return (size_t)g.B * g.Hq * g.max_splits * 2 * (g.d + 2);
}

// Records the first device-side error: later errors do not overwrite it.
__device__ inline void set_status(int32_t* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

__device__ inline float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ inline float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Bounded spin on an mbarrier phase.  Returns false if the wait gave up.
__device__ inline bool mbar_wait(uint32_t bar, uint32_t parity, long max_iter) {
  for (long i = 0; i < max_iter; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    if (ok) return true;
  }
  return false;
}

// The same, for waits that may be long: each poll lets the thread sleep up to ~0.25 us
// (woken early when the phase completes), so a waiting warp takes few issue slots.
__device__ inline bool mbar_wait_sleep(uint32_t bar, uint32_t parity, long max_iter) {
  for (long i = 0; i < max_iter; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(bar), "r"(parity), "r"(256) : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ inline void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ inline void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

// One-dimensional bulk copy global -> this CTA's shared memory, completing on
// `bar`.  No multicast.  dst, src and bytes must be multiples of 16.
__device__ inline void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Orders this thread's generic-proxy accesses of shared memory before later
// async-proxy (bulk copy) writes to it.
__device__ inline void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ inline uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

constexpr long kWaitIters = 1L << 24;   // bound of every device-side wait

// Tiled TMA load of a 3-D box into this CTA's shared memory, completing on `bar` (no
// multicast; the innermost coordinate times the element size must be a multiple of 16).
__device__ inline void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      :: "r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar) : "memory");
}

// cuTensorMapEncodeTiled from the driver (through the runtime's entry-point query); null if absent
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
constexpr int kMaxDevices = 64;

}  // namespace lvq

// Kernel launchers (defined in the .cu files, called by lvq_api.cu).
namespace lvq {
cudaError_t launch_pack(const Geo& g, const __nv_bfloat16* cb, __nv_bfloat16* cbp, float* cb_norm,
                        cudaStream_t s);
cudaError_t launch_rope_table(const Geo& g, float base, float* rope, cudaStream_t s);
cudaError_t launch_dequantize(const Geo& g, int layer, int step, int req, int kv, const uint8_t* idx,
                              const __nv_bfloat16* cbp, int tok_begin, int n_tok,
                              __nv_bfloat16* out, cudaStream_t s);
cudaError_t launch_encode_prefill(const Geo& g, int layer, int req, const __nv_bfloat16* kv,
                                  int64_t tok_stride, int kv_tokens, int tok_begin, int n_tok,
                                  int coded_offset, const __nv_bfloat16* cb, uint8_t* idx,
                                  int32_t* st, cudaStream_t s);
cudaError_t launch_encode_page(const Geo& g, int batch, const int32_t* ctx_len, int32_t* coded_len,
                               const __nv_bfloat16* ring, const __nv_bfloat16* cb, const float* cb_norm,
                               uint8_t* idx, int32_t* st, cudaStream_t s);
constexpr int kPageMaxBatch = 1024;     // requests one lvq_encode_page call can take
cudaError_t launch_kmeans_update(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                                 int kv_tokens, int tok_begin, int n_tok, int coded_offset, const uint8_t* idx,
                                 __nv_bfloat16* cb, uint32_t* counts, int32_t* st, cudaStream_t s);
cudaError_t launch_decode(const Geo& g, int layer, int step, int batch, const __nv_bfloat16* q,
                          const int32_t* ctx_len, const int32_t* coded_len,
                          const __nv_bfloat16* sink, const __nv_bfloat16* ring, const uint8_t* idx,
                          const __nv_bfloat16* cbp, const float* rope, int num_splits, float* ws,
                          float* out, float* lse, float* split_lse, int32_t* st, cudaStream_t s);
bool decode_supported(int d, int c);
int decode_bf16_capacity(int d, int c);
bool encode_tc_supported(int G, int c);
cudaError_t launch_encode_tc(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                             int kv_tokens, int tok_begin, int n_tok, int coded_offset,
                             const __nv_bfloat16* cb, uint8_t* idx, int32_t* st, cudaStream_t s);
bool encode_supported(int G, int c);
}  // namespace lvq
