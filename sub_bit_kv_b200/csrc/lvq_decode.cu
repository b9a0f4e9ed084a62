// Split-K decode attention over the LoopVQ coded cache, and the LSE merge.
//
// "LoopVQ summary", section "premises and limits": the attention kernel reads
// only the step-t slice of each codebook, splits the quantized tokens as in
// Flash-Decoding and merges them, and the bf16 sink/recent tokens, by
// logsumexp.  Section "how it differs": keys are stored before RoPE and RoPE is
// applied to the reconstructed key.
//
// Coded split (one CTA per (split, query head, request)):
//  * the step-t key slice of the head's codebooks, [256][n_g][c] bf16, is
//    bulk-copied into shared memory once (cp.async.bulk, no multicast);
//  * scores: lane (tq, P) of a warp owns pair-group P -- groups P and
//    P + n_g/2, i.e. the RoPE frequencies f = P*c + e, whose rotate-half
//    partners are channels f and f + d/2 -- and token slots tq, tq + 32/P', ...
//    of an 8-token page.  With z_f = q'_f + i q'_{f+d/2} (the query rotated at
//    its own position), the score of a key k at position p is
//      sum_f Re(z_f e^{-i p theta_f}) k_f + Im(z_f e^{-i p theta_f}) k_{f+d/2},
//    which equals q' . RoPE(k, p).  e^{-i p theta} is built from a per-page
//    factor (advanced by one complex multiply per page) times a per-slot
//    factor, all from fp64-built tables;
//  * values: instead of expanding every value, the softmax weight of a token is
//    added to a shared-memory histogram H[code][g] per group; after the split
//    the partial output is o[g*c + e] = sum_k H[k][g] * V_slice[k][g][e].
//    Weights use a reference maximum m_ref fixed per split and raised only if
//    a chunk's maximum exceeds it by 2^16 (then H is rescaled);
//  * the bf16 tokens (sink and recent window) form one more partial, computed
//    by a CTA of their own with an online softmax.
// Partials (o, m, l) go to the workspace; the merge kernel combines them.
#include "lvq_common.cuh"

namespace lvq {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kPagesPerWarp = 4;
constexpr int kChunk = kPage * kDecWarps * kPagesPerWarp;   // 256 coded tokens per chunk
static_assert(kChunk == kDecThreads, "one score per thread per chunk");
constexpr float kRescaleLog2 = 16.f;

template <int D, int C>
struct Dec {
  static constexpr int F = D / 2;        // RoPE frequencies
  static constexpr int NG = D / C;       // groups per step
  static constexpr int NP = NG / 2;      // pair-groups (groups g, g + NG/2)
  static constexpr int TQ = 32 / NP;     // token slots covered by one pass of a warp
  static constexpr int TPL = kPage / TQ; // K-side tokens per lane per page
  static constexpr int TPV = 32 / NG;    // V-side: lanes sharing a group (histogram copies)
  static constexpr int VPL = kPage / TPV;
  static constexpr int KS_BYTES = kEntries * D * 2;
  static constexpr int H_FLOATS = kEntries * 32;
  static constexpr int SMEM = KS_BYTES + H_FLOATS * 4 + kChunk * 4 + 2 * F * 4 + 64 * 4 + 16;
  static_assert(NP >= 4 && NP <= 32 && 32 % NP == 0, "pair-group mapping");
  static_assert(NG <= 32 && 32 % NG == 0, "histogram mapping");
};

__device__ inline float2 cmul(float2 a, float2 b) {
  return make_float2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ inline float2 cconj(float2 a) { return make_float2(a.x, -a.y); }

// e^{i p theta_f} from the coarse (8k) and fine (r < 8) tables.
__device__ inline float2 rope_at(const float* rope, int RC, int F, int p, int f) {
  const float2 a = reinterpret_cast<const float2*>(rope)[(size_t)(p >> 3) * F + f];
  const float2 b = reinterpret_cast<const float2*>(rope)[(size_t)(RC + (p & 7)) * F + f];
  return cmul(a, b);
}

__device__ inline int byte_of(uint2 w, int t) {
  return (int)(((t < 4 ? w.x : w.y) >> (8 * (t & 3))) & 0xffu);
}

template <int C>
__device__ inline void load_entry(const __nv_bfloat16* ks, int off, float (&k)[C]) {
  if constexpr (C == 4) {
    uint2 w = *reinterpret_cast<const uint2*>(ks + off);
    k[0] = bf16_lo(w.x); k[1] = bf16_hi(w.x); k[2] = bf16_lo(w.y); k[3] = bf16_hi(w.y);
  } else {
#pragma unroll
    for (int q = 0; q < C / 8; ++q) {
      uint4 w = *reinterpret_cast<const uint4*>(ks + off + 8 * q);
      k[8 * q + 0] = bf16_lo(w.x); k[8 * q + 1] = bf16_hi(w.x);
      k[8 * q + 2] = bf16_lo(w.y); k[8 * q + 3] = bf16_hi(w.y);
      k[8 * q + 4] = bf16_lo(w.z); k[8 * q + 5] = bf16_hi(w.z);
      k[8 * q + 6] = bf16_lo(w.w); k[8 * q + 7] = bf16_hi(w.w);
    }
  }
}

__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide reduction through red[kDecWarps]; every thread gets the result.
template <bool MAX>
__device__ inline float block_reduce(float v, float* red) {
  v = MAX ? warp_max(v) : warp_sum(v);
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kDecWarps; ++i) r = MAX ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

__device__ inline void write_partial(float* p, int D, const float* o, float m, float l) {
  for (int e = threadIdx.x; e < D; e += blockDim.x) p[e] = o ? o[e] : 0.f;
  if (threadIdx.x == 0) { p[D] = m; p[D + 1] = l; }
}

template <int D, int C>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(
    Geo g, int layer, int step, const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ ctx_len,
    const int32_t* __restrict__ coded_len, const __nv_bfloat16* __restrict__ sink,
    const __nv_bfloat16* __restrict__ ring, const uint8_t* __restrict__ idx,
    const __nv_bfloat16* __restrict__ cbp, const float* __restrict__ rope, int ns,
    float* __restrict__ ws, int32_t* st) {
  using X = Dec<D, C>;
  constexpr int F = X::F, NG = X::NG, NP = X::NP, TQ = X::TQ, TPL = X::TPL, TPV = X::TPV, VPL = X::VPL;
  extern __shared__ __align__(128) unsigned char smem[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(smem);
  float* Hs = reinterpret_cast<float*>(smem + X::KS_BYTES);
  float* sc = Hs + X::H_FLOATS;
  float2* zq = reinterpret_cast<float2*>(sc + kChunk);
  float* red = reinterpret_cast<float*>(zq + F);
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 64);

  const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int h = hq / (g.Hq / g.H);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blk = step / g.Tc, s = step % g.Tc;
  float* part = ws + (((size_t)b * g.Hq + hq) * (g.max_splits + 1) + j) * (D + 2);

  const int ctx = ctx_len[b], Lc = coded_len[b];
  const int S_eff = min(g.S, max(ctx, 0));
  const int recent = ctx - S_eff - Lc;
  const bool bad = ctx < 1 || ctx > g.max_ctx || Lc < 0 || Lc > g.P * kPage ||
                   (Lc > 0 && ctx < g.S + Lc) || recent < 0 || recent > g.R;
  if (bad) {
    if (j == 0 && tid == 0) set_status(st, LVQ_ECAPACITY);
    write_partial(part, D, nullptr, -INFINITY, 0.f);
    return;
  }

  // query rotated at its own position, scaled so scores come out in log2 units
  const int qpos = ctx - 1;
  const float qscale = 1.4426950408889634f * rsqrtf((float)D);
  const __nv_bfloat16* qv = q + ((size_t)b * g.Hq + hq) * D;
  for (int f = tid; f < F; f += blockDim.x) {
    float2 e = rope_at(rope, g.RC, F, qpos, f);
    float a = __bfloat162float(qv[f]), c2 = __bfloat162float(qv[f + F]);
    zq[f] = make_float2((a * e.x - c2 * e.y) * qscale, (c2 * e.x + a * e.y) * qscale);
  }

  if (j == ns) {
    // ---------------------------------------------------------------- bf16 partial
    constexpr int RF = F / 32;
    __syncthreads();
    float2 z[RF];
#pragma unroll
    for (int r = 0; r < RF; ++r) z[r] = zq[lane + 32 * r];
    float m = -INFINITY, l = 0.f, olo[RF], ohi[RF];
#pragma unroll
    for (int r = 0; r < RF; ++r) { olo[r] = 0.f; ohi[r] = 0.f; }
    const int nb = S_eff + recent;
    for (int i = warp; i < nb; i += kDecWarps) {
      int pos;
      size_t ko, vo;
      if (i < S_eff) {
        pos = i;
        ko = sink_off(g, layer, 0, step, b, h, i);
        vo = sink_off(g, layer, 1, step, b, h, i);
      } else {
        pos = g.S + Lc + (i - S_eff);
        const int slot = (pos - g.S) % g.R;
        ko = ring_off(g, layer, 0, step, b, h, slot);
        vo = ring_off(g, layer, 1, step, b, h, slot);
      }
      const __nv_bfloat16* kp = (i < S_eff ? sink : ring) + ko;
      const __nv_bfloat16* vp = (i < S_eff ? sink : ring) + vo;
      float part_s = 0.f;
#pragma unroll
      for (int r = 0; r < RF; ++r) {
        const int f = lane + 32 * r;
        float2 w = cmul(z[r], cconj(rope_at(rope, g.RC, F, pos, f)));
        part_s += w.x * __bfloat162float(kp[f]) + w.y * __bfloat162float(kp[f + F]);
      }
      const float sc2 = warp_sum(part_s);
      const float mn = fmaxf(m, sc2);
      const float alpha = exp2f(m - mn), p = exp2f(sc2 - mn);
      l = l * alpha + p;
#pragma unroll
      for (int r = 0; r < RF; ++r) {
        const int f = lane + 32 * r;
        olo[r] = olo[r] * alpha + p * __bfloat162float(vp[f]);
        ohi[r] = ohi[r] * alpha + p * __bfloat162float(vp[f + F]);
      }
      m = mn;
    }
    // combine the warps: sc[] holds m and l per warp, Hs holds o per warp
    if (lane == 0) { sc[warp] = m; sc[kDecWarps + warp] = l; }
#pragma unroll
    for (int r = 0; r < RF; ++r) {
      Hs[warp * D + lane + 32 * r] = olo[r];
      Hs[warp * D + F + lane + 32 * r] = ohi[r];
    }
    __syncthreads();
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sc[w]);
    if (M == -INFINITY) { write_partial(part, D, nullptr, -INFINITY, 0.f); return; }
    for (int e = tid; e < D; e += blockDim.x) {
      float o = 0.f;
      for (int w = 0; w < kDecWarps; ++w)
        if (sc[w] != -INFINITY) o += exp2f(sc[w] - M) * Hs[w * D + e];
      part[e] = o;
    }
    if (tid == 0) {
      float L = 0.f;
      for (int w = 0; w < kDecWarps; ++w)
        if (sc[w] != -INFINITY) L += exp2f(sc[w] - M) * sc[kDecWarps + w];
      part[D] = M;
      part[D + 1] = L;
    }
    return;
  }

  // ------------------------------------------------------------------ coded split j
  int chunk = (Lc + ns - 1) / ns;
  chunk = (chunk + 31) & ~31;
  const int n0 = min(Lc, j * chunk), n1 = min(Lc, n0 + chunk);
  if (n0 >= n1) { write_partial(part, D, nullptr, -INFINITY, 0.f); return; }

  const uint32_t bar_a = smem_addr(bar);
  if (tid == 0) {
    mbar_init(bar_a, 1);
    fence_mbar_init();
    mbar_expect_tx(bar_a, X::KS_BYTES);
    bulk_g2s(smem_addr(Ks), cbp + cbp_slice_off(g, layer, 0, blk, h, s), X::KS_BYTES, bar_a);
  }
  for (int i = tid; i < X::H_FLOATS; i += blockDim.x) Hs[i] = 0.f;
  __syncthreads();
  if (!mbar_wait(bar_a, 0, kWaitIters)) {
    set_status(st, LVQ_ETIMEOUT);
    mbar_wait(bar_a, 0, kWaitIters);   // let the copy land before the CTA exits
    write_partial(part, D, nullptr, -INFINITY, 0.f);
    return;
  }

  // per-lane constants of the score mapping
  const int P = lane % NP, tq = lane / NP;
  const int g_lo = P, g_hi = P + NP;
  float2 z[C], Et[TPL][C], stepc[C];
#pragma unroll
  for (int e = 0; e < C; ++e) {
    const int f = P * C + e;
    z[e] = zq[f];
    stepc[e] = cconj(rope_at(rope, g.RC, F, kPage * kDecWarps, f));
#pragma unroll
    for (int i = 0; i < TPL; ++i) Et[i][e] = cconj(rope_at(rope, g.RC, F, tq + TQ * i, f));
  }
  const int gv = lane % NG, tp = lane / NG;
  const uint8_t* page0 = idx + idx_page_off(g, layer, blk, b, h, 0);
  const __nv_bfloat16* Vs = cbp + cbp_slice_off(g, layer, 1, blk, h, s);

  float m_ref = -INFINITY, l_acc = 0.f;
  for (int c0 = n0; c0 < n1; c0 += kChunk) {
    // Phase A: scores of this chunk's tokens
    float2 u[C];
#pragma unroll
    for (int i = 0; i < kPagesPerWarp; ++i) {
      const int pl = warp + kDecWarps * i;
      const int tb = c0 + kPage * pl;
      if (tb >= n1) break;
      if (i == 0) {
#pragma unroll
        for (int e = 0; e < C; ++e) u[e] = cmul(z[e], cconj(rope_at(rope, g.RC, F, g.S + tb, P * C + e)));
      }
      const uint8_t* pg = page0 + (size_t)(tb >> 3) * g.page_bytes;
      const uint2 wlo = *reinterpret_cast<const uint2*>(pg + g_lo * kPage);
      const uint2 whi = *reinterpret_cast<const uint2*>(pg + g_hi * kPage);
      float acc[TPL];
#pragma unroll
      for (int i2 = 0; i2 < TPL; ++i2) {
        const int t = tq + TQ * i2;
        float klo[C], khi[C];
        load_entry<C>(Ks, (byte_of(wlo, t) * NG + g_lo) * C, klo);
        load_entry<C>(Ks, (byte_of(whi, t) * NG + g_hi) * C, khi);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < C; ++e) {
          const float2 w = cmul(u[e], Et[i2][e]);
          a = fmaf(w.x, klo[e], a);
          a = fmaf(w.y, khi[e], a);
        }
        acc[i2] = a;
      }
#pragma unroll
      for (int o = NP / 2; o > 0; o >>= 1) {
#pragma unroll
        for (int i2 = 0; i2 < TPL; ++i2) acc[i2] += __shfl_xor_sync(0xffffffffu, acc[i2], o);
      }
      if (P == 0) {
#pragma unroll
        for (int i2 = 0; i2 < TPL; ++i2) sc[pl * kPage + tq + TQ * i2] = acc[i2];
      }
#pragma unroll
      for (int e = 0; e < C; ++e) u[e] = cmul(u[e], stepc[e]);
    }
    __syncthreads();

    // Phase B: reference maximum and weights
    const bool valid = c0 + tid < n1;
    const float sv = valid ? sc[tid] : -INFINITY;
    const float mc = block_reduce<true>(sv, red);
    if (m_ref == -INFINITY) {
      m_ref = mc;
    } else if (mc > m_ref + kRescaleLog2) {
      const float f = exp2f(m_ref - mc);
      for (int i = tid; i < X::H_FLOATS; i += blockDim.x) Hs[i] *= f;
      l_acc *= f;
      m_ref = mc;
    }
    const float p = valid ? exp2f(sv - m_ref) : 0.f;
    l_acc += p;
    sc[tid] = p;
    __syncthreads();

    // Phase D: histogram of weights per (code, group)
#pragma unroll
    for (int i = 0; i < kPagesPerWarp; ++i) {
      const int pl = warp + kDecWarps * i;
      const int tb = c0 + kPage * pl;
      if (tb >= n1) break;
      const uint8_t* pg = page0 + (size_t)(tb >> 3) * g.page_bytes + NG * kPage;
      const uint2 wv = *reinterpret_cast<const uint2*>(pg + gv * kPage);
#pragma unroll
      for (int jv = 0; jv < VPL; ++jv) {
        const int t = tp + TPV * jv;
        if (tb + t < n1) atomicAdd(&Hs[(byte_of(wv, t) * TPV + tp) * NG + gv], sc[pl * kPage + t]);
      }
    }
    __syncthreads();
  }

  const float l_tot = block_reduce<false>(l_acc, red);
  // o[e] = sum_k H[k][g] V[k][g][e mod c], g = e / c
  constexpr int NKQ = kDecThreads / D;
  {
    const int e = tid % D, kq = tid / D, grp = e / C, ee = e % C;
    float o = 0.f;
    for (int k = kq; k < kEntries; k += NKQ) {
      float hsum = 0.f;
#pragma unroll
      for (int t2 = 0; t2 < TPV; ++t2) hsum += Hs[(k * TPV + t2) * NG + grp];
      o = fmaf(hsum, __bfloat162float(Vs[((size_t)k * NG + grp) * C + ee]), o);
    }
    sc[tid] = o;
  }
  __syncthreads();
  for (int e = tid; e < D; e += blockDim.x) {
    float o = 0.f;
#pragma unroll
    for (int kq = 0; kq < NKQ; ++kq) o += sc[kq * D + e];
    part[e] = o;
  }
  if (tid == 0) { part[D] = m_ref; part[D + 1] = l_tot; }
}

// LSE merge of the num_splits + 1 partials of one (request, query head).
template <int D>
__global__ void decode_merge_kernel(Geo g, int ns, const float* __restrict__ ws, float* __restrict__ out,
                                    float* __restrict__ lse, float* __restrict__ split_lse) {
  const int hq = blockIdx.x, b = blockIdx.y;
  const float* base = ws + ((size_t)b * g.Hq + hq) * (g.max_splits + 1) * (D + 2);
  float M = -INFINITY;
  for (int j = 0; j <= ns; ++j) {
    const float* p = base + (size_t)j * (D + 2);
    const float l = p[D + 1];
    if (l > 0.f) M = fmaxf(M, p[D] + log2f(l));
  }
  float den = 0.f;
  for (int j = 0; j <= ns; ++j) {
    const float* p = base + (size_t)j * (D + 2);
    const float l = p[D + 1];
    if (l > 0.f) den += exp2f(p[D] + log2f(l) - M);
  }
  const float L2 = M + log2f(den);
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float o = 0.f;
    for (int j = 0; j <= ns; ++j) {
      const float* p = base + (size_t)j * (D + 2);
      if (p[D + 1] > 0.f) o = fmaf(exp2f(p[D] - L2), p[e], o);
    }
    out[((size_t)b * g.Hq + hq) * D + e] = o;
  }
  if (threadIdx.x == 0) {
    constexpr float kLn2 = 0.6931471805599453f;
    lse[(size_t)b * g.Hq + hq] = L2 * kLn2;
    if (split_lse) {
      for (int j = 0; j <= ns; ++j) {
        const float* p = base + (size_t)j * (D + 2);
        const float l = p[D + 1];
        split_lse[((size_t)b * g.Hq + hq) * (ns + 1) + j] = l > 0.f ? (p[D] + log2f(l)) * kLn2 : -INFINITY;
      }
    }
  }
}

template <int D, int C>
static cudaError_t decode_as(const Geo& g, int layer, int step, int batch, const __nv_bfloat16* q,
                             const int32_t* ctx_len, const int32_t* coded_len, const __nv_bfloat16* sink,
                             const __nv_bfloat16* ring, const uint8_t* idx, const __nv_bfloat16* cbp,
                             const float* rope, int ns, float* ws, float* out, float* lse,
                             float* split_lse, int32_t* st, cudaStream_t s) {
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return ge;
  if (dev < 0 || dev >= kMaxDevices || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Dec<D, C>::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) attr_set[dev] = true;
  }
  dim3 grid(ns + 1, g.Hq, batch);
  decode_split_kernel<D, C><<<grid, kDecThreads, Dec<D, C>::SMEM, s>>>(
      g, layer, step, q, ctx_len, coded_len, sink, ring, idx, cbp, rope, ns, ws, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<D><<<dim3(g.Hq, batch), D, 0, s>>>(g, ns, ws, out, lse, split_lse);
  return cudaGetLastError();
}

bool decode_supported(int d, int c) {
  return (d == 128 && (c == 4 || c == 8 || c == 16)) || (d == 64 && (c == 4 || c == 8));
}

cudaError_t launch_decode(const Geo& g, int layer, int step, int batch, const __nv_bfloat16* q,
                          const int32_t* ctx_len, const int32_t* coded_len,
                          const __nv_bfloat16* sink, const __nv_bfloat16* ring, const uint8_t* idx,
                          const __nv_bfloat16* cbp, const float* rope, int num_splits, float* ws,
                          float* out, float* lse, float* split_lse, int32_t* st, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
#define LVQ_DEC(DD, CC)                                                                            \
  if (g.d == DD && g.c == CC)                                                                      \
    return decode_as<DD, CC>(g, layer, step, batch, q, ctx_len, coded_len, sink, ring, idx, cbp, rope, \
                             num_splits, ws, out, lse, split_lse, st, s);
  LVQ_DEC(128, 4) LVQ_DEC(128, 8) LVQ_DEC(128, 16) LVQ_DEC(64, 4) LVQ_DEC(64, 8)
#undef LVQ_DEC
  return cudaErrorInvalidValue;
}

}  // namespace lvq
