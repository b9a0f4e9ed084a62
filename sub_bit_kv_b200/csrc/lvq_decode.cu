// Split-K decode attention over the LoopVQ coded cache, with the LSE merge
// fused into the same launch.
//
// "LoopVQ summary", section "premises and limits": the attention kernel reads
// only the step-t slice of each codebook, splits the quantized tokens as in
// Flash-Decoding and merges them, and the bf16 sink/recent tokens, by
// logsumexp.  Section "how it differs": keys are stored before RoPE and RoPE is
// applied to the reconstructed key.
//
// One CTA per (split, query head, request), 16 warps:
//  * the step-t key slice of the head's codebooks, [256][n_g][c] bf16, is
//    bulk-copied into shared memory once (cp.async.bulk, no multicast);
//  * the split's code pages stream through a 3-stage shared-memory ring, one
//    bulk copy per 512-token chunk issued two chunks ahead;
//  * scores: lane (tq, P) owns pair-group P -- groups P and P + n_g/2, i.e. the
//    RoPE frequencies f = P*c + e whose rotate-half partners are channels f
//    and f + d/2 -- and every (32/n_p)-th token of its warp's pages.  With
//    z_f = q'_f + i q'_{f+d/2} (the query rotated at its own position), a key
//    k at position p scores
//      sum_f Re(z_f e^{-i p theta_f}) k_f + Im(z_f e^{-i p theta_f}) k_{f+d/2}
//    = q' . RoPE(k, p).  Along a lane's tokens (stride s) the factor
//    W_n = z e^{-i p_n theta} obeys W_{n+1} = 2 cos(s theta) W_n - W_{n-1}, so
//    each token costs one packed f32x2 FMA per frequency for the rotation and
//    one for the dot product; the recurrence is reseeded exactly every chunk;
//  * values: the softmax weight of a token is added to a shared-memory
//    histogram H[code][g]; the split's output is o[g*c + e] =
//    sum_k H[k][g] * V_slice[k][g][e].  Weights use a reference maximum fixed
//    per split, raised (and H rescaled) only if a chunk's maximum exceeds it
//    by 2^16;
//  * CTA ns (one more per request and head) computes the bf16 tokens'
//    partial: sink and recent window staged in shared memory by bulk copies,
//    scores with 4 threads per token, one softmax, P.V with a thread per
//    channel;
//  * the last CTA of a (request, head) to finish merges all partials by LSE
//    (a counter in the workspace, reset by that CTA).
#include "lvq_common.cuh"

namespace lvq {

constexpr int kDecWarps = 16;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kPPW = 4;                                    // pages per warp per chunk
constexpr int kChunk = kPage * kDecWarps * kPPW;           // 512 coded tokens per chunk
constexpr int kStages = 3;
static_assert(kChunk == kDecThreads, "one score per thread per chunk");
constexpr float kRescaleLog2 = 16.f;

template <int D, int C>
struct Dec {
  static constexpr int F = D / 2;          // RoPE frequencies
  static constexpr int NG = D / C;         // groups per step
  static constexpr int NP = NG / 2;        // pair-groups (groups g, g + NG/2)
  static constexpr int TQ = 32 / NP;       // token phases per page
  static constexpr int TPL = kPage / TQ;   // tokens per lane per page
  static constexpr int TPV = 32 / NG;      // V side: lanes per group
  static constexpr int VPL = kPage / TPV;
  static constexpr int PAGE = 2 * NG * kPage;
  static constexpr int STAGE = (kChunk / kPage) * PAGE;
  static constexpr int KS = kEntries * D * 2;
  static constexpr int HF = kEntries * 32;
  static constexpr int OFF_H = KS;
  static constexpr int OFF_RING = OFF_H + HF * 4;
  static constexpr int OFF_SC = OFF_RING + kStages * STAGE;
  static constexpr int OFF_ZQ = OFF_SC + kChunk * 4;
  static constexpr int OFF_RED = OFF_ZQ + F * 8;
  static constexpr int OFF_BAR = OFF_RED + 64 * 4;
  static constexpr int SMEM = OFF_BAR + 8 * (kStages + 1) + 16;
  static_assert(NP >= 4 && NP <= 32 && 32 % NP == 0, "pair-group mapping");
  static_assert(NG <= 32 && 32 % NG == 0, "histogram mapping");
  static_assert(SMEM <= 227 * 1024, "shared memory");
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
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kDecWarps; ++i) r = MAX ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

// k_lo and k_hi entries of one group pair -> packed (k_lo[e], k_hi[e]) fp32 pairs
template <int C>
__device__ inline void load_pairs(const unsigned char* ks, uint32_t off_lo, uint32_t off_hi, float2 (&kp)[C]) {
  uint32_t lo[C / 2], hi[C / 2];
  if constexpr (C == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(ks + off_lo);
    const uint2 b = *reinterpret_cast<const uint2*>(ks + off_hi);
    lo[0] = a.x; lo[1] = a.y; hi[0] = b.x; hi[1] = b.y;
  } else {
#pragma unroll
    for (int q = 0; q < C / 8; ++q) {
      const uint4 a = *reinterpret_cast<const uint4*>(ks + off_lo + 16 * q);
      const uint4 b = *reinterpret_cast<const uint4*>(ks + off_hi + 16 * q);
      lo[4 * q + 0] = a.x; lo[4 * q + 1] = a.y; lo[4 * q + 2] = a.z; lo[4 * q + 3] = a.w;
      hi[4 * q + 0] = b.x; hi[4 * q + 1] = b.y; hi[4 * q + 2] = b.z; hi[4 * q + 3] = b.w;
    }
  }
#pragma unroll
  for (int w = 0; w < C / 2; ++w) {
    kp[2 * w] = make_float2(bf16_lo(lo[w]), bf16_lo(hi[w]));
    kp[2 * w + 1] = make_float2(bf16_hi(lo[w]), bf16_hi(hi[w]));
  }
}

__device__ inline void store_partial(float* p, int D, float o_e, int e, float m, float l) {
  if (e >= 0) p[e] = o_e;
  if (threadIdx.x == 0) { p[D] = m; p[D + 1] = l; }
}

template <int D, int C>
__global__ void __launch_bounds__(kDecThreads, 1) decode_kernel(
    Geo g, int layer, int step, const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ ctx_len,
    const int32_t* __restrict__ coded_len, const __nv_bfloat16* __restrict__ sink,
    const __nv_bfloat16* __restrict__ ring, const uint8_t* __restrict__ idx,
    const __nv_bfloat16* __restrict__ cbp, const float* __restrict__ rope, int ns,
    float* __restrict__ ws, float* __restrict__ out, float* __restrict__ lse, float* __restrict__ split_lse,
    int32_t* st) {
  using X = Dec<D, C>;
  constexpr int F = X::F, NG = X::NG, NP = X::NP, TQ = X::TQ, TPL = X::TPL, TPV = X::TPV, VPL = X::VPL;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* Ks = smem;
  float* Hs = reinterpret_cast<float*>(smem + X::OFF_H);
  unsigned char* ringb = smem + X::OFF_RING;
  float* sc = reinterpret_cast<float*>(smem + X::OFF_SC);
  float2* zq = reinterpret_cast<float2*>(smem + X::OFF_ZQ);
  float* red = reinterpret_cast<float*>(smem + X::OFF_RED);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);   // [0]: K slice, [1..]: ring stages

  const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int h = hq / (g.Hq / g.H);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blk = step / g.Tc, s = step % g.Tc;
  const size_t slot_base = ((size_t)b * g.Hq + hq) * (g.max_splits + 1);
  float* part = ws + (slot_base + j) * (D + 2);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + (size_t)g.B * g.Hq * (g.max_splits + 1) * (D + 2));

  const int ctx = ctx_len[b], Lc = coded_len[b];
  const int S_eff = min(g.S, max(ctx, 0));
  const int recent = ctx - S_eff - Lc;
  const bool bad = ctx < 1 || ctx > g.max_ctx || Lc < 0 || Lc > g.P * kPage ||
                   (Lc > 0 && ctx < g.S + Lc) || recent < 0 || recent > g.R;

  int chunk = (Lc + ns - 1) / ns;
  chunk = (chunk + 31) & ~31;
  const int n0 = bad ? 0 : min(Lc, j * chunk), n1 = bad ? 0 : min(Lc, n0 + chunk);
  const bool do_coded = n0 < n1;

  // ---- start the bulk copies: key slice, then the first two chunks of pages
  const uint32_t bar0 = smem_addr(&bars[0]);
  const uint8_t* pages = idx + idx_page_off(g, layer, blk, b, h, 0);
  const int n_chunks = do_coded ? (n1 - n0 + kChunk - 1) / kChunk : 0;
  auto issue_chunk = [&](int ci) {
    const int c0 = n0 + ci * kChunk;
    const int np = (min(n1, c0 + kChunk) - c0 + kPage - 1) / kPage;
    const uint32_t bar = smem_addr(&bars[1 + ci % kStages]);
    mbar_expect_tx(bar, np * X::PAGE);
    bulk_g2s(smem_addr(ringb + (ci % kStages) * X::STAGE), pages + (size_t)(c0 / kPage) * X::PAGE,
             np * X::PAGE, bar);
  };
  if (tid == 0 && do_coded) {
    for (int i = 0; i <= kStages; ++i) mbar_init(smem_addr(&bars[i]), 1);
    fence_mbar_init();
    mbar_expect_tx(bar0, X::KS);
    bulk_g2s(smem_addr(Ks), cbp + cbp_slice_off(g, layer, 0, blk, h, s), X::KS, bar0);
    for (int ci = 0; ci < min(2, n_chunks); ++ci) issue_chunk(ci);
  }

  if (bad && j == 0 && tid == 0) set_status(st, LVQ_ECAPACITY);

  // ---- query rotated at its own position, scaled so scores come out in log2 units
  if (!bad) {
    const int qpos = ctx - 1;
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    const __nv_bfloat16* qv = q + ((size_t)b * g.Hq + hq) * D;
    for (int f = tid; f < F; f += blockDim.x) {
      const float2 e = rope_at(rope, g.RC, F, qpos, f);
      const float a = __bfloat162float(qv[f]), c2 = __bfloat162float(qv[f + F]);
      zq[f] = make_float2((a * e.x - c2 * e.y) * qscale, (c2 * e.x + a * e.y) * qscale);
    }
  }
  for (int i = tid; i < X::HF; i += blockDim.x) Hs[i] = 0.f;
  __syncthreads();

  float m_ref = -INFINITY, l_acc = 0.f;
  bool timed_out = false;
  if (do_coded) {
    // every wait is bounded; the outcome is made block-uniform before acting on it
    if (__syncthreads_or(!mbar_wait(bar0, 0, kWaitIters))) timed_out = true;

    // lane constants: pair-group P, token phase tq
    const int P = lane % NP, tq = lane / NP;
    const int g_lo = P, g_hi = P + NP;
    float2 z[C], twoc[C], etq[C], echunk[C], U[C];
    const int p_first = g.S + n0 + kPage * kPPW * warp + tq;   // the lane's first token position
#pragma unroll
    for (int e = 0; e < C; ++e) {
      const int f = P * C + e;
      z[e] = zq[f];
      const float2 r = rope_at(rope, g.RC, F, TQ, f);
      twoc[e] = make_float2(2.f * r.x, 2.f * r.x);
      etq[e] = cconj(r);
      echunk[e] = cconj(rope_at(rope, g.RC, F, kChunk, f));
      U[e] = cmul(z[e], cconj(rope_at(rope, g.RC, F, p_first, f)));
    }
    const int gv = lane % NG, tp = lane / NG;
    // byte selector for __byte_perm: result byte 0 = group offset byte, byte 1 = code, bytes 2-3 = 0
    const uint32_t gb_lo = (uint32_t)g_lo * C * 2, gb_hi = (uint32_t)g_hi * C * 2;
    static_assert(D * 2 == 256 || D * 2 == 128, "key row stride");

    for (int ci = 0; ci < n_chunks && !timed_out; ++ci) {
      const int c0 = n0 + ci * kChunk;
      const uint32_t bar = smem_addr(&bars[1 + ci % kStages]);
      if (__syncthreads_or(!mbar_wait(bar, (ci / kStages) & 1, kWaitIters))) {
        timed_out = true;
        if (tid == 0)   // let the copies still in flight land before the CTA can exit
          for (int k = ci; k < min(n_chunks, ci + 2); ++k)
            mbar_wait(smem_addr(&bars[1 + k % kStages]), (k / kStages) & 1, kWaitIters);
        break;
      }
      const unsigned char* stage = ringb + (ci % kStages) * X::STAGE;

      // Phase A: scores of the warp's 4 contiguous pages
      {
        float2 Wc[C], Wn[C];
#pragma unroll
        for (int e = 0; e < C; ++e) { Wc[e] = U[e]; Wn[e] = cmul(U[e], etq[e]); }
#pragma unroll
        for (int pi = 0; pi < kPPW; ++pi) {
          const int pl = warp * kPPW + pi;
          const int tb = c0 + kPage * pl;
          float acc[TPL];
          if (tb < n1) {
            const unsigned char* pg = stage + pl * X::PAGE;
            const uint2 wlo = *reinterpret_cast<const uint2*>(pg + g_lo * kPage);
            const uint2 whi = *reinterpret_cast<const uint2*>(pg + g_hi * kPage);
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
              const int t = tq + TQ * i;
              const uint32_t clo = ((t < 4 ? wlo.x : wlo.y) >> (8 * (t & 3))) & 0xffu;
              const uint32_t chi = ((t < 4 ? whi.x : whi.y) >> (8 * (t & 3))) & 0xffu;
              float2 kp[C];
              load_pairs<C>(Ks, clo * (D * 2) + gb_lo, chi * (D * 2) + gb_hi, kp);
              float2 a2 = __fmul2_rn(Wc[0], kp[0]);
#pragma unroll
              for (int e = 1; e < C; ++e) a2 = __ffma2_rn(Wc[e], kp[e], a2);
              acc[i] = a2.x + a2.y;
#pragma unroll
              for (int e = 0; e < C; ++e) {
                const float2 nx = __ffma2_rn(twoc[e], Wn[e], make_float2(-Wc[e].x, -Wc[e].y));
                Wc[e] = Wn[e];
                Wn[e] = nx;
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < TPL; ++i) acc[i] = 0.f;
          }
          // transposed reduction over the NP lanes of a token phase
          int cnt = TPL;
#pragma unroll
          for (int o = NP / 2; o > 0; o >>= 1) {
            if (cnt > 1) {
              const int half = cnt / 2;
              const bool up = (lane & o) != 0;
#pragma unroll
              for (int k = 0; k < TPL / 2; ++k) {
                if (k < half) {
                  const float send = up ? acc[k] : acc[k + half];
                  const float keep = up ? acc[k + half] : acc[k];
                  acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
              }
              cnt = half;
            } else {
              acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], o);
            }
          }
          constexpr int GRP = NP / TPL;        // lanes holding the same total
          if ((P % GRP) == 0) sc[pl * kPage + tq + TQ * (P / GRP)] = acc[0];
        }
      }
      __syncthreads();

      // Phase B: reference maximum and weights
      const bool valid = c0 + tid < n1;
      const float sv = valid ? sc[tid] : -INFINITY;
      const float mc = block_reduce<true>(sv, red);
      if (m_ref == -INFINITY) {
        m_ref = mc;
      } else if (mc > m_ref + kRescaleLog2) {
        const float fct = exp2f(m_ref - mc);
        for (int i = tid; i < X::HF; i += blockDim.x) Hs[i] *= fct;
        l_acc *= fct;
        m_ref = mc;
      }
      const float p = valid ? exp2f(sv - m_ref) : 0.f;
      l_acc += p;
      sc[tid] = p;
      __syncthreads();

      // Phase D: histogram of the weights per (code, group)
#pragma unroll
      for (int pi = 0; pi < kPPW; ++pi) {
        const int pl = warp * kPPW + pi;
        if (c0 + kPage * pl >= n1) break;
        const unsigned char* pg = stage + pl * X::PAGE + NG * kPage;
        const uint2 wv = *reinterpret_cast<const uint2*>(pg + gv * kPage);
#pragma unroll
        for (int jv = 0; jv < VPL; ++jv) {
          const int t = tp + TPV * jv;
          const uint32_t code = ((t < 4 ? wv.x : wv.y) >> (8 * (t & 3))) & 0xffu;
          atomicAdd(&Hs[(code * TPV + tp) * NG + gv], sc[pl * kPage + t]);
        }
      }
      __syncthreads();
      // refill the stage consumed in the previous chunk
      if (tid == 0 && ci + 2 < n_chunks) issue_chunk(ci + 2);
#pragma unroll
      for (int e = 0; e < C; ++e) U[e] = cmul(U[e], echunk[e]);
    }
    if (timed_out) {
      if (tid == 0) {
        set_status(st, LVQ_ETIMEOUT);
        mbar_wait(bar0, 0, kWaitIters);
      }
      m_ref = -INFINITY;
      l_acc = 0.f;
    }
  }

  // ---- coded partial: o[e] = sum_k H[k][g] V[k][g][e mod c]
  if (j < ns) {
    const float l_tot = block_reduce<false>(l_acc, red);
    constexpr int NKQ = kDecThreads / D;
    const int e = tid % D, kq = tid / D, grp = e / C, ee = e % C;
    float o = 0.f;
    if (do_coded) {
      const __nv_bfloat16* Vs = cbp + cbp_slice_off(g, layer, 1, blk, h, s) + (size_t)grp * C + ee;
#pragma unroll 8
      for (int k = kq; k < kEntries; k += NKQ) {
        float hsum = 0.f;
#pragma unroll
        for (int t2 = 0; t2 < TPV; ++t2) hsum += Hs[(k * TPV + t2) * NG + grp];
        o = fmaf(hsum, __bfloat162float(Vs[(size_t)k * D]), o);
      }
    }
    sc[tid] = o;
    __syncthreads();
    float oe = 0.f;
    if (tid < D) {
#pragma unroll
      for (int k2 = 0; k2 < NKQ; ++k2) oe += sc[k2 * D + tid];
    }
    store_partial(part, D, oe, tid < D ? tid : -1, do_coded ? m_ref : -INFINITY, do_coded ? l_tot : 0.f);
  }

  // ---- CTA ns: the bf16 partial (sink tokens and recent window)
  if (j == ns) {
    float* pb = ws + (slot_base + ns) * (D + 2);
    const int nb = bad ? 0 : S_eff + recent;
    // stage sink K/V and the whole recent-window ring K/V for (layer, step, b, h)
    __nv_bfloat16* Kb = reinterpret_cast<__nv_bfloat16*>(smem);                 // [S + R][D]
    __nv_bfloat16* Vb = Kb + (size_t)(g.S + g.R) * D;                            // [S + R][D]
    bool ok = true;
    if (nb > 0) {
      const uint32_t barb = smem_addr(&bars[0]);
      if (tid == 0) {
        mbar_init(barb, 1);
        fence_mbar_init();
        const uint32_t sb = (uint32_t)S_eff * D * 2, rb = (uint32_t)g.R * D * 2;
        mbar_expect_tx(barb, 2 * (sb + rb));
        if (sb) {
          bulk_g2s(smem_addr(Kb), sink + sink_off(g, layer, 0, step, b, h, 0), sb, barb);
          bulk_g2s(smem_addr(Vb), sink + sink_off(g, layer, 1, step, b, h, 0), sb, barb);
        }
        bulk_g2s(smem_addr(Kb + (size_t)g.S * D), ring + ring_off(g, layer, 0, step, b, h, 0), rb, barb);
        bulk_g2s(smem_addr(Vb + (size_t)g.S * D), ring + ring_off(g, layer, 1, step, b, h, 0), rb, barb);
      }
      __syncthreads();
      ok = !__syncthreads_or(!mbar_wait(barb, 0, kWaitIters));
      if (!ok && tid == 0) set_status(st, LVQ_ETIMEOUT);
    }
    // scores: 4 threads per token, each a quarter of the frequencies
    constexpr int FQ = F / 4;
    for (int i0 = 0; i0 < nb && ok; i0 += kDecThreads / 4) {
      const int i = i0 + tid / 4, qf = tid % 4;
      float part_s = 0.f;
      if (i < nb) {
        int pos, row;
        if (i < S_eff) { pos = i; row = i; }
        else { pos = g.S + Lc + (i - S_eff); row = g.S + (pos - g.S) % g.R; }
        const __nv_bfloat16* kr = Kb + (size_t)row * D;
#pragma unroll 4
        for (int f = qf * FQ; f < (qf + 1) * FQ; ++f) {
          const float2 w = cmul(zq[f], cconj(rope_at(rope, g.RC, F, pos, f)));
          part_s = fmaf(w.x, __bfloat162float(kr[f]), part_s);
          part_s = fmaf(w.y, __bfloat162float(kr[f + F]), part_s);
        }
      }
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 1);
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 2);
      if (i < nb && qf == 0) sc[i] = part_s;
    }
    __syncthreads();
    float mloc = -INFINITY;
    for (int i = tid; i < nb && ok; i += kDecThreads) mloc = fmaxf(mloc, sc[i]);
    const float M = block_reduce<true>(mloc, red);
    float lloc = 0.f;
    for (int i = tid; i < nb && ok; i += kDecThreads) {
      const float p = exp2f(sc[i] - M);
      sc[i] = p;
      lloc += p;
    }
    const float Lb = block_reduce<false>(lloc, red);     // block_reduce syncs: sc holds the weights
    constexpr int NTS = kDecThreads / D;
    const int e = tid % D, ts = tid / D;
    float o = 0.f;
    for (int i = ts; i < nb && ok; i += NTS) {
      const int row = i < S_eff ? i : g.S + (Lc + (i - S_eff)) % g.R;
      o = fmaf(sc[i], __bfloat162float(Vb[(size_t)row * D + e]), o);
    }
    __syncthreads();
    Hs[ts * D + e] = o;    // after the barrier nothing reads the staged tokens any more
    __syncthreads();
    if (tid < D) {
      float oe = 0.f;
#pragma unroll
      for (int k2 = 0; k2 < NTS; ++k2) oe += Hs[k2 * D + tid];
      pb[tid] = oe;
    }
    if (tid == 0) {
      const bool any = ok && nb > 0;
      pb[D] = any ? M : -INFINITY;
      pb[D + 1] = any ? Lb : 0.f;
    }
  }

  // ---- the last CTA of this (request, head) merges the ns + 1 partials
  __threadfence();
  __syncthreads();
  __shared__ int last;
  if (tid == 0) last = atomicAdd(&counters[(size_t)b * g.Hq + hq], 1) == ns;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* base = ws + slot_base * (D + 2);
  if (tid <= ns) {
    const float* pj = base + (size_t)tid * (D + 2);
    const float l = __ldcg(pj + D + 1);
    sc[tid] = l > 0.f ? __ldcg(pj + D) + log2f(l) : -INFINITY;   // lse2 of partial tid
  }
  __syncthreads();
  float M = -INFINITY;
  for (int i = 0; i <= ns; ++i) M = fmaxf(M, sc[i]);
  float den = 0.f;
  if (M != -INFINITY)
    for (int i = 0; i <= ns; ++i) den += exp2f(sc[i] - M);
  const float L2 = M == -INFINITY ? -INFINITY : M + log2f(den);
  if (tid < D) {
    float o = 0.f;
    if (M != -INFINITY)
      for (int i = 0; i <= ns; ++i) {
        const float* pj = base + (size_t)i * (D + 2);
        if (sc[i] != -INFINITY) o = fmaf(exp2f(__ldcg(pj + D) - L2), __ldcg(pj + tid), o);
      }
    out[((size_t)b * g.Hq + hq) * D + tid] = o;
  }
  constexpr float kLn2 = 0.6931471805599453f;
  if (tid == 0) {
    lse[(size_t)b * g.Hq + hq] = L2 * kLn2;
    counters[(size_t)b * g.Hq + hq] = 0;
  }
  if (split_lse && tid <= ns) split_lse[((size_t)b * g.Hq + hq) * (ns + 1) + tid] = sc[tid] * kLn2;
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
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Dec<D, C>::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) attr_set[dev] = true;
  }
  dim3 grid(ns + 1, g.Hq, batch);
  decode_kernel<D, C><<<grid, kDecThreads, Dec<D, C>::SMEM, s>>>(
      g, layer, step, q, ctx_len, coded_len, sink, ring, idx, cbp, rope, ns, ws, out, lse, split_lse, st);
  return cudaGetLastError();
}

// bf16 tokens (sink + ring slots) the bf16-partial CTA can stage: K and V must
// fit below the score buffer.
template <int D, int C>
static int bf16_capacity_as() { return Dec<D, C>::OFF_SC / (4 * D); }

int decode_bf16_capacity(int d, int c) {
  if (d == 128 && c == 4) return bf16_capacity_as<128, 4>();
  if (d == 128 && c == 8) return bf16_capacity_as<128, 8>();
  if (d == 128 && c == 16) return bf16_capacity_as<128, 16>();
  if (d == 64 && c == 4) return bf16_capacity_as<64, 4>();
  if (d == 64 && c == 8) return bf16_capacity_as<64, 8>();
  return 0;
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
#define LVQ_DEC(DD, CC)                                                                                \
  if (g.d == DD && g.c == CC)                                                                          \
    return decode_as<DD, CC>(g, layer, step, batch, q, ctx_len, coded_len, sink, ring, idx, cbp, rope, \
                             num_splits, ws, out, lse, split_lse, st, s);
  LVQ_DEC(128, 4) LVQ_DEC(128, 8) LVQ_DEC(128, 16) LVQ_DEC(64, 4) LVQ_DEC(64, 8)
#undef LVQ_DEC
  return cudaErrorInvalidValue;
}

}  // namespace lvq
