// Exact nearest-entry encoders: prefill (many tokens per codebook) and the
// decode-time page encode (8 tokens per codebook, every layer and step).
//
// "LoopVQ summary", section "how it differs": a joint vector holds c = G/Tc
// channels of each of the Tc steps of a block (keys before RoPE) and is
// encoded as its single nearest codebook entry.  Distances are the direct
// form sum_j (x_j - C_kj)^2 in fp64: differences and squares of bf16 values
// are exact there, so the index equals the exact nearest entry except when
// two entries are equally near to within fp64 rounding.  Ties go to the lowest
// index (strict '<' while scanning k upward).
#include "lvq_common.cuh"

namespace lvq {

constexpr int kEncThreads = 128;

// Grid: x = token tiles of kEncThreads, y = codebook (kv, blk, h, grp).
template <int G, int C>
__global__ void __launch_bounds__(kEncThreads) encode_prefill_kernel(
    Geo g, int layer, int req, const __nv_bfloat16* __restrict__ kv, int64_t tok_stride, int kv_tokens,
    int tok_begin, int n_tok, int coded_offset, const __nv_bfloat16* __restrict__ cb,
    uint8_t* __restrict__ idx) {
  constexpr int TC = G / C;
  __shared__ float cbs[kEntries * G];   // fp32 copies of the bf16 entries (exact)
  int cid = blockIdx.y;
  const int grp = cid % g.ng; cid /= g.ng;
  const int h = cid % g.H; cid /= g.H;
  const int blk = cid % g.nblk; cid /= g.nblk;
  const int kvi = cid;

  const __nv_bfloat16* Cb = cb + cb_off(g, layer, kvi, blk, h, grp);
  for (int i = threadIdx.x; i < kEntries * G; i += blockDim.x) cbs[i] = __bfloat162float(Cb[i]);
  __syncthreads();

  const int local = blockIdx.x * blockDim.x + threadIdx.x;
  if (local >= n_tok) return;
  const int n = tok_begin + local;

  double x[G];
  const int64_t step_stride = tok_stride * kv_tokens;
  const __nv_bfloat16* base = kv + ((int64_t)kvi * g.T) * step_stride + (int64_t)n * tok_stride +
                              (int64_t)h * g.d + grp * C;
#pragma unroll
  for (int s = 0; s < TC; ++s) {
    const __nv_bfloat16* p = base + (int64_t)(blk * TC + s) * step_stride;
#pragma unroll
    for (int e = 0; e < C; ++e) x[s * C + e] = (double)__bfloat162float(p[e]);
  }
  double best = 1e300;
  int bk = 0;
#pragma unroll 2
  for (int k = 0; k < kEntries; ++k) {
    const float* ce = cbs + k * G;
    double acc = 0.0;
#pragma unroll
    for (int j = 0; j < G; ++j) {
      double df = x[j] - (double)ce[j];
      acc = fma(df, df, acc);
    }
    if (acc < best) { best = acc; bk = k; }
  }
  const int cn = coded_offset + local;
  uint8_t* page = idx + idx_page_off(g, layer, blk, req, h, cn >> 3);
  page[kvi * g.ng * kPage + grp * kPage + (cn & 7)] = (uint8_t)bk;
}

template <int G, int C>
static cudaError_t encode_prefill_as(const Geo& g, int layer, int req, const __nv_bfloat16* kv,
                                     int64_t tok_stride, int kv_tokens, int tok_begin, int n_tok,
                                     int coded_offset, const __nv_bfloat16* cb, uint8_t* idx,
                                     cudaStream_t s) {
  dim3 grid((n_tok + kEncThreads - 1) / kEncThreads, 2 * g.nblk * g.H * g.ng);
  encode_prefill_kernel<G, C><<<grid, kEncThreads, 0, s>>>(g, layer, req, kv, tok_stride, kv_tokens,
                                                            tok_begin, n_tok, coded_offset, cb, idx);
  return cudaGetLastError();
}

bool encode_supported(int G, int c) {
  return (G == 16 || G == 32) && (c == 4 || c == 8 || c == 16) && c <= G;
}

cudaError_t launch_encode_prefill(const Geo& g, int layer, int req, const __nv_bfloat16* kv,
                                  int64_t tok_stride, int kv_tokens, int tok_begin, int n_tok,
                                  int coded_offset, const __nv_bfloat16* cb, uint8_t* idx,
                                  int32_t* st, cudaStream_t s) {
  (void)st;
  if (n_tok == 0) return cudaSuccess;
#define LVQ_ENC(GG, CC)                                                                          \
  if (g.G == GG && g.c == CC)                                                                    \
    return encode_prefill_as<GG, CC>(g, layer, req, kv, tok_stride, kv_tokens, tok_begin, n_tok, \
                                     coded_offset, cb, idx, s);
  LVQ_ENC(16, 4) LVQ_ENC(16, 8) LVQ_ENC(16, 16) LVQ_ENC(32, 4) LVQ_ENC(32, 8) LVQ_ENC(32, 16)
#undef LVQ_ENC
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------- page encode

// The request's recent window is full (R = n_recent + 8 tokens) exactly when
// its oldest page must be encoded.  Returns 1 to encode, 0 to skip, -1 on a
// capacity error.
__device__ inline int page_due(const Geo& g, int ctx, int coded) {
  int recent = ctx - g.S - coded;
  if (ctx > g.max_ctx || coded < 0 || recent > g.R) return -1;
  if (recent < g.R) return 0;
  if (coded + kPage > g.P * kPage) return -1;
  return 1;
}

// One warp per codebook (layer, kv, blk, h, grp) and request; lane l scans
// entries l, l+32, ..., then the warp takes the lexicographic (distance, k)
// minimum, which is the lowest index among equal distances.
constexpr int kPageWarps = 4;

__global__ void __launch_bounds__(32 * kPageWarps) encode_page_kernel(
    Geo g, const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ coded_len,
    const __nv_bfloat16* __restrict__ ring, const __nv_bfloat16* __restrict__ cb,
    uint8_t* __restrict__ idx, int32_t* st) {
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31;
  long cid = (long)blockIdx.x * kPageWarps + (threadIdx.x >> 5);
  const long n_cb = (long)g.L * 2 * g.nblk * g.H * g.ng;
  if (cid >= n_cb) return;
  const int ctx = ctx_len[b], coded = coded_len[b];
  const int due = page_due(g, ctx, coded);
  if (due < 0) { if (cid == 0 && lane == 0) set_status(st, LVQ_ECAPACITY); return; }
  if (due == 0) return;

  const int grp = (int)(cid % g.ng); cid /= g.ng;
  const int h = (int)(cid % g.H); cid /= g.H;
  const int blk = (int)(cid % g.nblk); cid /= g.nblk;
  const int kvi = (int)(cid % 2); cid /= 2;
  const int layer = (int)cid;

  // this lane's 8 entries, widened to fp64
  const __nv_bfloat16* C = cb + cb_off(g, layer, kvi, blk, h, grp);
  uint8_t* page_base = idx + idx_page_off(g, layer, blk, b, h, 0) + kvi * g.ng * kPage + grp * kPage;
  for (int t = 0; t < kPage; ++t) {
    const int cn = coded + t;
    const int slot = cn % g.R;           // position S + cn lives in slot (cn mod R)
    double x[32];
    for (int s = 0; s < g.Tc; ++s) {
      const __nv_bfloat16* p = ring + ring_off(g, layer, kvi, blk * g.Tc + s, b, h, slot) + grp * g.c;
      for (int e = 0; e < g.c; ++e) x[s * g.c + e] = (double)__bfloat162float(p[e]);
    }
    double best = 1e300;
    int bk = 0;
    for (int i = 0; i < kEntries / 32; ++i) {
      const int k = lane + 32 * i;
      const __nv_bfloat16* ce = C + (size_t)k * g.G;
      double acc = 0.0;
      for (int j = 0; j < g.G; ++j) {
        double df = x[j] - (double)__bfloat162float(ce[j]);
        acc = fma(df, df, acc);
      }
      if (acc < best) { best = acc; bk = k; }
    }
    for (int off = 16; off > 0; off >>= 1) {
      double ob = __shfl_xor_sync(0xffffffffu, best, off);
      int ok = __shfl_xor_sync(0xffffffffu, bk, off);
      if (ob < best || (ob == best && ok < bk)) { best = ob; bk = ok; }
    }
    if (lane == 0) page_base[(size_t)(cn >> 3) * g.page_bytes + (cn & 7)] = (uint8_t)bk;
  }
}

__global__ void advance_kernel(Geo g, int batch, const int32_t* __restrict__ ctx_len,
                               int32_t* __restrict__ coded_len) {
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    if (page_due(g, ctx_len[b], coded_len[b]) == 1) coded_len[b] += kPage;
  }
}

cudaError_t launch_encode_page(const Geo& g, int batch, const int32_t* ctx_len, int32_t* coded_len,
                               const __nv_bfloat16* ring, const __nv_bfloat16* cb, uint8_t* idx,
                               int32_t* st, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  const long n_cb = (long)g.L * 2 * g.nblk * g.H * g.ng;
  dim3 grid((unsigned)((n_cb + kPageWarps - 1) / kPageWarps), batch);
  encode_page_kernel<<<grid, 32 * kPageWarps, 0, s>>>(g, ctx_len, coded_len, ring, cb, idx, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  advance_kernel<<<1, 256, 0, s>>>(g, batch, ctx_len, coded_len);
  return cudaGetLastError();
}

}  // namespace lvq
