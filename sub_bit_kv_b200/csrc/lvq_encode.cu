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
  idx[idx_code_off(g, layer, blk, req, h, kvi, cn, grp)] = (uint8_t)bk;
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

// One CTA per codebook (layer, kv, blk, h, grp), looping over the requests whose
// page is due, so each codebook is read from memory once.  The codebook and
// its squared norms sit in shared memory; warp t takes token t of the page and
// lane l the entries l, l + 32, ...  Distances are first taken in the fp32
// expansion form n_k - 2 x.C_k; every entry within
// eps = 2^-14 (||x||^2 + max_k n_k) of the minimum is a candidate (the fp32
// error is far below eps), and when there are several the candidates are
// rescored exactly in the fp64 direct form, lowest index on ties.
constexpr int kPageThreads = 32 * kPage;

template <int G, int C>
__global__ void __launch_bounds__(kPageThreads, 2) encode_page_kernel(
    Geo g, int batch, const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ coded_len,
    const __nv_bfloat16* __restrict__ ring, const __nv_bfloat16* __restrict__ cb, uint8_t* __restrict__ idx,
    int32_t* st) {
  constexpr int TC = G / C;
  __shared__ float cbs[kEntries * G];     // fp32 copies of the bf16 entries (exact)
  __shared__ float nrm[kEntries];
  __shared__ float nmax_s;
  long cid = blockIdx.x;
  const int grp = (int)(cid % g.ng); cid /= g.ng;
  const int h = (int)(cid % g.H); cid /= g.H;
  const int blk = (int)(cid % g.nblk); cid /= g.nblk;
  const int kvi = (int)(cid % 2); cid /= 2;
  const int layer = (int)cid;
  const int tid = threadIdx.x, lane = tid & 31, t = tid >> 5;

  bool any = false;
  for (int b = 0; b < batch; ++b) any |= page_due(g, ctx_len[b], coded_len[b]) == 1;
  if (!any) return;

  const __nv_bfloat16* Cg = cb + cb_off(g, layer, kvi, blk, h, grp);
  for (int i = tid; i < kEntries * G; i += kPageThreads) cbs[i] = __bfloat162float(Cg[i]);
  if (tid == 0) nmax_s = 0.f;
  __syncthreads();
  {
    const int k = tid;                    // kPageThreads == kEntries
    double n = 0.0;
#pragma unroll
    for (int j = 0; j < G; ++j) n += (double)cbs[k * G + j] * (double)cbs[k * G + j];
    nrm[k] = (float)n;
    atomicMax(reinterpret_cast<int*>(&nmax_s), __float_as_int((float)n));
  }
  __syncthreads();

  for (int b = 0; b < batch; ++b) {
    const int ctx = ctx_len[b], coded = coded_len[b];
    const int due = page_due(g, ctx, coded);
    if (due < 0) {
      if (blockIdx.x == 0 && tid == 0) set_status(st, LVQ_ECAPACITY);
      continue;
    }
    if (due == 0) continue;
    const int cn = coded + t;             // this warp's token, coded slot cn
    const int slot = cn % g.R;            // position S + cn lives in slot (cn mod R)
    float x[G];
    float xx = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < TC; ++s2) {
      const __nv_bfloat16* p = ring + ring_off(g, layer, kvi, blk * TC + s2, b, h, slot) + grp * C;
#pragma unroll
      for (int e = 0; e < C; ++e) {
        x[s2 * C + e] = __bfloat162float(p[e]);
        xx = fmaf(x[s2 * C + e], x[s2 * C + e], xx);
      }
    }
    float dv[kEntries / 32];
    float best = INFINITY;
#pragma unroll
    for (int i = 0; i < kEntries / 32; ++i) {
      const float* ce = cbs + (lane + 32 * i) * G;
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < G; ++j) dot = fmaf(x[j], ce[j], dot);
      dv[i] = fmaf(-2.f, dot, nrm[lane + 32 * i]);
      best = fminf(best, dv[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = fminf(best, __shfl_xor_sync(0xffffffffu, best, o));
    const float thr = best + ldexpf(xx + nmax_s, -14);
    int n_cand = 0, k_cand = kEntries;
#pragma unroll
    for (int i = 0; i < kEntries / 32; ++i)
      if (dv[i] <= thr) { ++n_cand; k_cand = min(k_cand, lane + 32 * i); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_cand += __shfl_xor_sync(0xffffffffu, n_cand, o);
      k_cand = min(k_cand, __shfl_xor_sync(0xffffffffu, k_cand, o));
    }
    int code = k_cand;
    if (n_cand > 1) {
      // near-tie: exact fp64 direct-form distances of the candidates, lowest index on ties
      double bd = 1e300;
      int bk = kEntries;
#pragma unroll 1
      for (int i = 0; i < kEntries / 32; ++i) {
        if (dv[i] <= thr) {
          const int k = lane + 32 * i;
          double acc = 0.0;
#pragma unroll
          for (int j = 0; j < G; ++j) {
            const double df = (double)x[j] - (double)cbs[k * G + j];
            acc = fma(df, df, acc);
          }
          if (acc < bd) { bd = acc; bk = k; }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, bd, o);
        const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
        if (ob < bd || (ob == bd && ok < bk)) { bd = ob; bk = ok; }
      }
      code = bk;
    }
    if (lane == 0) {
      idx[idx_code_off(g, layer, blk, b, h, kvi, cn, grp)] = (uint8_t)code;
    }
  }
}

__global__ void advance_kernel(Geo g, int batch, const int32_t* __restrict__ ctx_len,
                               int32_t* __restrict__ coded_len) {
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    if (page_due(g, ctx_len[b], coded_len[b]) == 1) coded_len[b] += kPage;
  }
}

template <int G, int C>
static cudaError_t encode_page_as(const Geo& g, int batch, const int32_t* ctx_len, int32_t* coded_len,
                                  const __nv_bfloat16* ring, const __nv_bfloat16* cb, uint8_t* idx, int32_t* st,
                                  cudaStream_t s) {
  const long n_cb = (long)g.L * 2 * g.nblk * g.H * g.ng;
  encode_page_kernel<G, C><<<(unsigned)n_cb, kPageThreads, 0, s>>>(g, batch, ctx_len, coded_len, ring, cb, idx, st);
  return cudaGetLastError();
}

cudaError_t launch_encode_page(const Geo& g, int batch, const int32_t* ctx_len, int32_t* coded_len,
                               const __nv_bfloat16* ring, const __nv_bfloat16* cb, uint8_t* idx,
                               int32_t* st, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  cudaError_t e = cudaErrorInvalidValue;
#define LVQ_PG(GG, CC) \
  if (g.G == GG && g.c == CC) e = encode_page_as<GG, CC>(g, batch, ctx_len, coded_len, ring, cb, idx, st, s);
  LVQ_PG(16, 4) LVQ_PG(16, 8) LVQ_PG(16, 16) LVQ_PG(32, 4) LVQ_PG(32, 8) LVQ_PG(32, 16)
#undef LVQ_PG
  if (e != cudaSuccess) return e;
  advance_kernel<<<1, 256, 0, s>>>(g, batch, ctx_len, coded_len);
  return cudaGetLastError();
}

}  // namespace lvq
