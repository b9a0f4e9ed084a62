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
// live in shared memory.  Tiles of 128 tokens stream in by TMA through a
// 3-stage ring: the tokens' bf16 values of the item's channels ([Tc][128][64/Tc],
// a 3-D box of the K/V tensor) and the code pages that hold their codes (a 3-D
// box of the index rows).  A token of an item is 64 elements (Tc steps x the
// set's channels, or equivalently 64/G joint vectors): two passes of a warp,
// each lane adding one value to its entry's sum with a shared-memory fp64
// atomic.  After the last tile the CTA divides, rounds and writes its entries.
#include "lvq_common.cuh"

namespace lvq {

namespace km {

constexpr int kThreads = 512;
constexpr int kElems = 64;               // elements of one token of an item
constexpr int kTile = 128;               // tokens per tile
constexpr int kStages = 3;
constexpr int kTilePages = kTile / kPage + 1;   // a tile that starts inside a page spans one more

template <int G, int C>
struct Km {
  static constexpr int TC = G / C;                 // steps per block
  static constexpr int GS = kElems / G;            // groups per item
  static constexpr int CH = GS * C;                // channels per step of an item
  // accumulators [GS][256][G], group gi shifted by 4 doubles so that the groups of one
  // warp pass start in different banks
  static constexpr int ACC = GS * kEntries * G + 4 * GS;
  static constexpr int RAW = TC * kTile * CH * 2;              // [TC][kTile][CH] bf16
  static constexpr int CODES = kTilePages * GS * kPage;        // [kTilePages][GS][8] code bytes
  static constexpr int STAGE = RAW + (CODES + 127) / 128 * 128;
  static constexpr int OFF_CNT = ACC * 8;
  static constexpr int OFF_STAGE = (OFF_CNT + GS * kEntries * 4 + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = OFF_STAGE + kStages * STAGE;
  static constexpr int SMEM = OFF_BAR + 8 * kStages + 1024;    // + alignment slack of the base
  static_assert(TC * CH == kElems, "one token of an item is 64 elements");
  static_assert((CH * 2) % 16 == 0 && (GS * kPage) % 16 == 0, "TMA boxes of whole 16-byte units");
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
    const __grid_constant__ CUtensorMap kv_map, const __grid_constant__ CUtensorMap code_map, Geo g, int layer,
    int req, int tok_begin, int n_tok, int coded_offset, __nv_bfloat16* cb, uint32_t* counts, int32_t* st) {
  using X = Km<G, C>;
  constexpr int TC = X::TC, GS = X::GS, CH = X::CH;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  double* acc_s = reinterpret_cast<double*>(smem);                      // [GS][256][G] (+ offsets)
  uint32_t* cnt_s = reinterpret_cast<uint32_t*>(smem + X::OFF_CNT);     // [GS][256]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_sets = g.ng / GS;
  int it = blockIdx.x;
  const int gset = it % n_sets; it /= n_sets;
  const int h = it % g.H; it /= g.H;
  const int blk = it % g.nblk; it /= g.nblk;
  const int kvi = it;
  const int stream = (((layer * g.nblk + blk) * g.B + req) * g.H + h) * 2 + kvi;   // index-row stream
  const int n_tiles = (n_tok + kTile - 1) / kTile;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(smem_addr(&bars[i]), 1);
    fence_mbar_init();
  }
  for (int i = tid; i < X::ACC; i += kThreads) acc_s[i] = 0.0;
  for (int i = tid; i < GS * kEntries; i += kThreads) cnt_s[i] = 0u;
  __syncthreads();

  auto issue = [&](int tl) {             // one thread: the tile's values and code pages
    if ((g.fault & kFaultKmeansDropTile) && tl == 0) return;   // test hook: this copy never happens
    unsigned char* stg = smem + X::OFF_STAGE + (tl % kStages) * X::STAGE;
    const uint32_t bar = smem_addr(&bars[tl % kStages]);
    mbar_expect_tx(bar, X::RAW + X::CODES);
    tma_load_3d(smem_addr(stg), &kv_map, h * g.d + gset * CH, tok_begin + tl * kTile, kvi * g.T + blk * TC, bar);
    tma_load_3d(smem_addr(stg + X::RAW), &code_map, gset * GS * kPage, (coded_offset + tl * kTile) >> 3, stream,
                bar);
  };
  if (tid == 0)
    for (int tl = 0; tl < min(kStages, n_tiles); ++tl) issue(tl);

  // element el of a token (pass p = el / 32): step s = el / CH, channel ch = el % CH of the
  // item's channels, group gi = ch / C, joint-vector element j = s * C + ch % C
  int s_of[2], ch_of[2], gi_of[2], j_of[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const int el = p * 32 + lane;
    s_of[p] = el / CH;
    ch_of[p] = el % CH;
    gi_of[p] = ch_of[p] / C;
    j_of[p] = s_of[p] * C + ch_of[p] % C;
  }

  bool failed = false;
  int tl = 0;
  for (; tl < n_tiles; ++tl) {
    const unsigned char* stg = smem + X::OFF_STAGE + (tl % kStages) * X::STAGE;
    if (__syncthreads_or(!mbar_wait(smem_addr(&bars[tl % kStages]), (tl / kStages) & 1u, g.wait_iters))) {
      failed = true;
      break;
    }
    const __nv_bfloat16* vals = reinterpret_cast<const __nv_bfloat16*>(stg);    // [TC][kTile][CH]
    const unsigned char* cpg = stg + X::RAW;                                      // [pages][GS][8]
    const int cn0 = coded_offset + tl * kTile;
    const int n_here = min(kTile, n_tok - tl * kTile);
    for (int r = warp; r < n_here; r += kThreads / 32) {
      const int cn = cn0 + r;
      const int prow = (cn >> 3) - (cn0 >> 3);
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int gi = gi_of[p];
        const int a = cpg[(prow * GS + gi) * kPage + (cn & 7)];
        const float x = __bfloat162float(vals[(s_of[p] * kTile + r) * CH + ch_of[p]]);
        atomicAdd(&acc_s[(gi * kEntries + a) * G + j_of[p] + 4 * gi], (double)x);
        if (j_of[p] == 0) atomicAdd(&cnt_s[gi * kEntries + a], 1u);
      }
    }
    fence_proxy_async_shared();      // this thread's reads of the stage before its refill by TMA
    __syncthreads();
    if (tid == 0 && tl + kStages < n_tiles) issue(tl + kStages);
  }
  if (failed) {
    // every issued copy lands before the CTA can exit
    if (tid == 0) {
      set_status(st, LVQ_ETIMEOUT);
      for (int t2 = tl; t2 < min(n_tiles, tl + kStages); ++t2)
        mbar_wait(smem_addr(&bars[t2 % kStages]), (t2 / kStages) & 1u, g.wait_iters);
    }
    __syncthreads();
    return;
  }

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
                                    __nv_bfloat16* cb, uint32_t* counts, int32_t* st, cudaStream_t s) {
  using X = Km<G, C>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap kv_map, code_map;
  {  // values: channels of a token row, tokens, (K/V, step) planes
    cuuint64_t dims[3] = {(cuuint64_t)g.H * g.d, (cuuint64_t)kv_tokens, (cuuint64_t)2 * g.T};
    cuuint64_t strides[2] = {(cuuint64_t)tok_stride * 2, (cuuint64_t)tok_stride * kv_tokens * 2};
    cuuint32_t box[3] = {(cuuint32_t)X::CH, (cuuint32_t)kTile, (cuuint32_t)X::TC};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(kv), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {  // code pages: bytes of a page, pages of a stream, streams (layer, block, request, head, K/V)
    const cuuint64_t n_streams = (cuuint64_t)g.L * g.nblk * g.B * g.H * 2;
    cuuint64_t dims[3] = {(cuuint64_t)g.page_bytes, (cuuint64_t)g.P, n_streams};
    cuuint64_t strides[2] = {(cuuint64_t)g.page_bytes, (cuuint64_t)g.P * g.page_bytes};
    cuuint32_t box[3] = {(cuuint32_t)(X::GS * kPage), (cuuint32_t)kTilePages, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&code_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(idx), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
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
  kmeans_update_kernel<G, C><<<items, kThreads, X::SMEM, s>>>(kv_map, code_map, g, layer, req, tok_begin, n_tok,
                                                              coded_offset, cb, counts, st);
  return cudaGetLastError();
}

}  // namespace km

cudaError_t launch_kmeans_update(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                                 int kv_tokens, int tok_begin, int n_tok, int coded_offset, const uint8_t* idx,
                                 __nv_bfloat16* cb, uint32_t* counts, int32_t* st, cudaStream_t s) {
#define LVQ_KM(GG, CC)                                                                                     \
  if (g.G == GG && g.c == CC)                                                                              \
    return km::kmeans_update_as<GG, CC>(g, layer, req, kv, tok_stride, kv_tokens, tok_begin, n_tok,        \
                                        coded_offset, idx, cb, counts, st, s);
  LVQ_KM(16, 4) LVQ_KM(16, 8) LVQ_KM(16, 16) LVQ_KM(32, 4) LVQ_KM(32, 8) LVQ_KM(32, 16)
#undef LVQ_KM
  return cudaErrorInvalidValue;
}

}  // namespace lvq
