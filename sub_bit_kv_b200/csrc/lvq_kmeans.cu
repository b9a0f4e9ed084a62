// Codebook construction: the update step of plain k-means over joint vectors.
//
// "LoopVQ summary", section "how it differs": the codebooks are initialised by
// k-means over the loop-axis joint vectors (Fisher-weighted there; the weights
// need a model's gradients, so this is the unweighted form).  Section "premises
// and limits": k-means over the calibration tokens is the first calibration stage.
//
// One Lloyd iteration is the assignment -- the exact nearest entry, which the
// prefill encoder already computes into the index rows -- followed by this
// update: every entry moves to the mean of the joint vectors coded with it, and
// an entry no vector chose keeps its value.  The new entries are stored in bf16,
// rounded once from the fp64 mean (to nearest, ties to even).
//
// Exactness: the sums are accumulated in fp64.  A sum of bf16 values is exact
// in fp64 unless the values of one sum span more than about 53 - 8 - log2(count)
// binades, so the accumulation order does not change it, and the fp64 division
// and the single rounding to bf16 give the same entry as an fp64 computation of
// the mean on the host.
//
// CTA: one item = (K/V, block, head, a set of 64/G groups), all tokens.  The
// item's accumulators ([64/G][256][G] fp64, 128 KB, and [64/G][256] counts)
// live in shared memory.  A token of an item is 64 elements (Tc steps x the
// set's channels, or equivalently 64/G joint vectors): two passes of a warp,
// each lane loading one bf16 value (lanes of one step read contiguous channels)
// and adding it to its entry's sum with a shared-memory fp64 atomic.  After the
// last token the CTA divides, rounds and writes its entries.
#include "lvq_common.cuh"

namespace lvq {

namespace km {

constexpr int kThreads = 512;
constexpr int kElems = 64;               // elements of one token of an item

template <int G, int C>
struct Km {
  static constexpr int TC = G / C;                 // steps per block
  static constexpr int GS = kElems / G;            // groups per item
  static constexpr int CH = GS * C;                // channels per step of an item
  // accumulators [GS][256][G], group gi shifted by 4 doubles so that the groups of one
  // warp pass start in different banks
  static constexpr int ACC = GS * kEntries * G + 4 * GS;
  static constexpr int SMEM = ACC * 8 + GS * kEntries * 4;
  static_assert(TC * CH == kElems, "one token of an item is 64 elements");
  static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");
};

// fp64 -> bf16, rounded once to nearest with ties to even: scale so that one bf16 step
// at |v| is 1, round to an integer, scale back (exact: the result is a bf16 value), then
// convert that exact value.  bf16 steps are 2^(e-8) for |v| in [2^(e-1), 2^e), and 2^-133
// below the normal range.
__device__ inline __nv_bfloat16 bf16_rne_from_f64(double v) {
  if (v == 0.0 || !isfinite(v)) return __float2bfloat16_rn((float)v);
  int e;
  frexp(v, &e);
  const int se = max(e - 8, -133);
  const double r = ldexp(rint(ldexp(v, -se)), se);
  return __float2bfloat16_rn((float)r);     // r is a bf16 value (or beyond the range: inf)
}

template <int G, int C>
__global__ void __launch_bounds__(kThreads, 1) kmeans_update_kernel(
    Geo g, int layer, int req, const __nv_bfloat16* __restrict__ kv, int64_t tok_stride, int64_t plane,
    int tok_begin, int n_tok, int coded_offset, const uint8_t* __restrict__ idx, __nv_bfloat16* cb,
    uint32_t* counts) {
  using X = Km<G, C>;
  constexpr int TC = X::TC, GS = X::GS, CH = X::CH;
  extern __shared__ double acc_s[];                                  // [GS][256][G] (+ offsets)
  uint32_t* cnt_s = reinterpret_cast<uint32_t*>(acc_s + X::ACC);     // [GS][256]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_sets = g.ng / GS;
  int it = blockIdx.x;
  const int gset = it % n_sets; it /= n_sets;
  const int h = it % g.H; it /= g.H;
  const int blk = it % g.nblk; it /= g.nblk;
  const int kvi = it;

  for (int i = tid; i < X::ACC; i += kThreads) acc_s[i] = 0.0;
  for (int i = tid; i < GS * kEntries; i += kThreads) cnt_s[i] = 0u;
  __syncthreads();

  // element el of a token (pass p = el / 32): step s = el / CH, channel ch = el % CH of the
  // item's channels, group gi = ch / C, joint-vector element j = s * C + ch % C
  int s_of[2], gi_of[2], j_of[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int el = p * 32 + lane;
    s_of[p] = el / CH;
    const int ch = el % CH;
    gi_of[p] = ch / C;
    j_of[p] = s_of[p] * C + ch % C;
  }
  const int ch0 = gset * CH;                   // first channel of the item in a step row
  const uint8_t* codes = idx + idx_stream_off(g, layer, blk, req, h, kvi);
  const __nv_bfloat16* xb = kv + (int64_t)(kvi * g.T + blk * TC) * plane + (int64_t)h * g.d + ch0;

  for (int t = warp; t < n_tok; t += kThreads / 32) {
    const int n = tok_begin + t, cn = coded_offset + t;
    const uint8_t* cpage = codes + (size_t)(cn >> 3) * g.page_bytes + (cn & 7);
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const int gi = gi_of[p];
      const int a = cpage[(gset * GS + gi) * kPage];
      const float x = __bfloat162float(xb[(int64_t)s_of[p] * plane + (int64_t)n * tok_stride + (p * 32 + lane) % CH]);
      atomicAdd(&acc_s[(gi * kEntries + a) * G + j_of[p] + 4 * gi], (double)x);
      if (j_of[p] == 0) atomicAdd(&cnt_s[gi * kEntries + a], 1u);
    }
  }
  __syncthreads();

  // entry k of group gi moves to its mean; entries no vector chose keep their value
  for (int i = tid; i < GS * kEntries * G; i += kThreads) {
    const int gi = i / (kEntries * G), k = (i / G) % kEntries, j = i % G;
    const uint32_t cnt = cnt_s[gi * kEntries + k];
    if (cnt > 0) {
      const double mean = acc_s[(gi * kEntries + k) * G + j + 4 * gi] / (double)cnt;
      cb[cb_off(g, layer, kvi, blk, h, gset * GS + gi) + (size_t)k * G + j] = bf16_rne_from_f64(mean);
    }
  }
  if (counts)
    for (int i = tid; i < GS * kEntries; i += kThreads) {
      const int gi = i / kEntries, k = i % kEntries;
      counts[((((size_t)kvi * g.nblk + blk) * g.H + h) * g.ng + gset * GS + gi) * kEntries + k] = cnt_s[i];
    }
}

template <int G, int C>
static cudaError_t kmeans_update_as(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                                    int kv_tokens, int tok_begin, int n_tok, int coded_offset, const uint8_t* idx,
                                    __nv_bfloat16* cb, uint32_t* counts, cudaStream_t s) {
  using X = Km<G, C>;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kmeans_update_kernel<G, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, X::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int items = 2 * g.nblk * g.H * (g.ng / X::GS);
  kmeans_update_kernel<G, C><<<items, kThreads, X::SMEM, s>>>(g, layer, req, kv, tok_stride,
                                                              tok_stride * (int64_t)kv_tokens, tok_begin, n_tok,
                                                              coded_offset, idx, cb, counts);
  return cudaGetLastError();
}

}  // namespace km

cudaError_t launch_kmeans_update(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                                 int kv_tokens, int tok_begin, int n_tok, int coded_offset, const uint8_t* idx,
                                 __nv_bfloat16* cb, uint32_t* counts, cudaStream_t s) {
#define LVQ_KM(GG, CC)                                                                                     \
  if (g.G == GG && g.c == CC)                                                                              \
    return km::kmeans_update_as<GG, CC>(g, layer, req, kv, tok_stride, kv_tokens, tok_begin, n_tok,        \
                                        coded_offset, idx, cb, counts, s);
  LVQ_KM(16, 4) LVQ_KM(16, 8) LVQ_KM(16, 16) LVQ_KM(32, 4) LVQ_KM(32, 8) LVQ_KM(32, 16)
#undef LVQ_KM
  return cudaErrorInvalidValue;
}

}  // namespace lvq
