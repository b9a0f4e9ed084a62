// Split-K decode attention over the LoopVQ coded cache, with the LSE merge
// fused into the same launch.
//
// "LoopVQ summary", section "premises and limits": the attention kernel reads
// only the step-t slice of each codebook, splits the quantized tokens as in
// Flash-Decoding and merges them, and the bf16 sink/recent tokens, by
// logsumexp.  Section "how it differs": keys are stored before RoPE and RoPE is
// applied to the reconstructed key.
//
// Grid (num_splits + 1, query heads, requests); 15 compute warps and one
// producer warp per CTA, one CTA per SM.
//  * Coded split j < num_splits: the producer bulk-copies the step-t key slice
//    of the head's codebooks ([256][n_g][c] bf16, one contiguous span) and then
//    the split's code pages, 480 tokens per chunk, through a 3-stage ring
//    (cp.async.bulk into shared memory, no multicast; full/empty mbarriers).
//  * Scores: lane (tq, P) of a compute warp owns pair-group P -- groups P and
//    P + n_g/2, i.e. the RoPE frequencies f = P*c + e whose rotate-half
//    partners are channels f and f + d/2 -- and every (32/n_p)-th token of the
//    warp's pages.  With z_f = q'_f + i q'_{f+d/2} (the query rotated at its own
//    position), a key k at position p scores
//      sum_f Re(z_f e^{-i p theta_f}) k_f + Im(z_f e^{-i p theta_f}) k_{f+d/2}
//    = q' . RoPE(k, p).  Along a lane's tokens (stride s) the factor
//    W_n = z e^{-i p_n theta} obeys W_{n+1} = 2 cos(s theta) W_n - W_{n-1}: one
//    packed f32x2 FMA per frequency for the rotation and one for the dot
//    product; the recurrence is reseeded exactly at every chunk.  A code byte
//    becomes its shared-memory row address in one byte permute.
//  * Values: each token's weight 2^(s - m_ref) is added to a shared-memory
//    histogram H[code][g] (conflict-free red.shared); the split's output is
//    o[g*c + e] = sum_k H[k][g] V_slice[k][g][e].  m_ref is the maximum over
//    each warp's first page; if any later score exceeds it by more than 2^64
//    the split is recomputed with its true maximum (exact, rare).
//  * CTA num_splits computes the bf16 tokens' partial (sink and recent window)
//    from shared-memory copies.
//  * The last CTA of a (request, head) to finish merges the partials by LSE
//    (a counter in the workspace, returned to zero by that CTA).
#include "lvq_common.cuh"

namespace lvq {

constexpr int kCW = 15;                      // compute warps (+1 producer: 512 threads, 128 registers)
constexpr int kCT = 32 * kCW;                // compute threads
constexpr int kThr = kCT + 32;               // + producer warp
constexpr int kPPW = 4;                      // pages per warp per chunk
constexpr int kChunk = kPage * kCW * kPPW;   // 480 coded tokens per chunk
constexpr int kStages = 3;
constexpr float kGuardLog2 = 64.f;           // largest s - m_ref accepted without recomputation

template <int D, int C>
struct Dec {
  static constexpr int F = D / 2;          // RoPE frequencies
  static constexpr int NG = D / C;         // groups per step
  static constexpr int NP = NG / 2;        // pair-groups (groups g, g + NG/2)
  static constexpr int TQ = 32 / NP;       // token phases per page
  static constexpr int TPL = kPage / TQ;   // tokens per lane per page
  static constexpr int GRP = NP / TPL;     // lanes holding the same reduced score
  static constexpr int TPV = 32 / NG;      // V side: lanes per group
  static constexpr int VPL = kPage / TPV;
  static constexpr int PAGE = 2 * NG * kPage;
  static constexpr int STAGE = (kChunk / kPage) * PAGE;
  static constexpr int KS = kEntries * D * 2;
  static constexpr int HF = kEntries * 32;
  static constexpr int OFF_H = KS;
  static constexpr int OFF_RING = OFF_H + HF * 4;
  static constexpr int OFF_SC = OFF_RING + kStages * STAGE;      // bf16 CTA: scores of its tokens
  static constexpr int SC_N = 512;
  static constexpr int OFF_PW = OFF_SC + SC_N * 4;                // per-warp token weights
  static constexpr int OFF_ZQ = OFF_PW + kCW * kPage * 4;
  static constexpr int OFF_RED = OFF_ZQ + F * 8;
  static constexpr int OFF_MISC = OFF_RED + 64 * 4;
  static constexpr int OFF_BAR = OFF_MISC + 16;
  static constexpr int SMEM = OFF_BAR + 8 * (2 * kStages + 1) + 8;
  static_assert(NP >= 4 && NP <= 32 && 32 % NP == 0, "pair-group mapping");
  static_assert(NG <= 32 && 32 % NG == 0, "histogram mapping");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(OFF_SC % 16 == 0 && OFF_RING % 16 == 0, "alignment");
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

// Reduction over all threads of the CTA through red[]; every thread gets the
// result.  Threads without data pass the identity.
template <bool MAX>
__device__ inline float block_reduce(float v, float* red) {
  v = MAX ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) r = MAX ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

__device__ inline void compute_sync() { asm volatile("bar.sync 1, %0;" :: "n"(kCT) : "memory"); }

__device__ inline void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

// Per-lane state of the score mapping.
template <int D, int C>
struct Lane {
  int P, tq, g_lo, g_hi;
  uint32_t gb_lo, gb_hi;              // byte offsets of the lane's groups inside a key-slice row
  uint32_t sel[2];                    // byte-permute selectors for the lane's token bytes
  float2 z[C], twoc[C], etq[C];
};

template <int D, int C>
__device__ inline void lane_init(Lane<D, C>& L, int lane, const float2* zq, const float* rope, int RC) {
  using X = Dec<D, C>;
  constexpr int NP = X::NP, TQ = X::TQ, F = X::F;
  L.P = lane % NP;
  L.tq = lane / NP;
  L.g_lo = L.P;
  L.g_hi = L.P + NP;
  L.gb_lo = (uint32_t)L.g_lo * C * 2;
  L.gb_hi = (uint32_t)L.g_hi * C * 2;
  // byte permute: result byte 0 = the group offset byte (second operand, byte 0),
  // byte 1 = the token's code byte (first operand), bytes 2-3 = zero (second operand, byte 1)
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int bpos = (L.tq + 2 * k * (TQ == 2 ? 1 : 0)) & 3;
    L.sel[k] = 0x5504u | ((uint32_t)bpos << 4);
  }
#pragma unroll
  for (int e = 0; e < C; ++e) {
    const int f = L.P * C + e;
    L.z[e] = zq[f];
    const float2 r = rope_at(rope, RC, F, TQ, f);
    L.twoc[e] = make_float2(2.f * r.x, 2.f * r.x);
    L.etq[e] = cconj(r);
  }
}

// Scores of the 8 tokens of one page.  On return the lane holds the score of
// token t_own = tq + TQ * (P / GRP) (every GRP-th lane of a phase has it); W
// advances by TPL tokens.
template <int D, int C>
__device__ inline float page_scores(const Lane<D, C>& L, const unsigned char* Ks, const unsigned char* pg,
                                    float2 (&Wc)[C], float2 (&Wn)[C]) {
  using X = Dec<D, C>;
  constexpr int TQ = X::TQ, TPL = X::TPL, NP = X::NP;
  const uint2 wlo = *reinterpret_cast<const uint2*>(pg + L.g_lo * kPage);
  const uint2 whi = *reinterpret_cast<const uint2*>(pg + L.g_hi * kPage);
  float acc[TPL];
#pragma unroll
  for (int i = 0; i < TPL; ++i) {
    // the word holding token t = tq + TQ*i: compile-time unless TQ == 8
    uint32_t xl, xh, sel;
    if constexpr (TQ == 8) {
      xl = L.tq < 4 ? wlo.x : wlo.y;
      xh = L.tq < 4 ? whi.x : whi.y;
      sel = L.sel[0];
    } else {
      const int word = (TQ * i) / 4;
      xl = word ? wlo.y : wlo.x;
      xh = word ? whi.y : whi.x;
      sel = L.sel[(TQ * i / 2) & 1];
    }
    uint32_t off_lo, off_hi;
    if constexpr (D * 2 == 256) {
      // row address = code * 256 + group offset, in one byte permute
      off_lo = __byte_perm(xl, L.gb_lo, sel);
      off_hi = __byte_perm(xh, L.gb_hi, sel);
    } else {
      off_lo = (__byte_perm(xl, 0u, sel) >> 8) * (D * 2) + L.gb_lo;
      off_hi = (__byte_perm(xh, 0u, sel) >> 8) * (D * 2) + L.gb_hi;
    }
    uint32_t lo[C / 2], hi[C / 2];
    if constexpr (C == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(Ks + off_lo);
      const uint2 b = *reinterpret_cast<const uint2*>(Ks + off_hi);
      lo[0] = a.x; lo[1] = a.y; hi[0] = b.x; hi[1] = b.y;
    } else {
#pragma unroll
      for (int q = 0; q < C / 8; ++q) {
        const uint4 a = *reinterpret_cast<const uint4*>(Ks + off_lo + 16 * q);
        const uint4 b = *reinterpret_cast<const uint4*>(Ks + off_hi + 16 * q);
        lo[4 * q + 0] = a.x; lo[4 * q + 1] = a.y; lo[4 * q + 2] = a.z; lo[4 * q + 3] = a.w;
        hi[4 * q + 0] = b.x; hi[4 * q + 1] = b.y; hi[4 * q + 2] = b.z; hi[4 * q + 3] = b.w;
      }
    }
    float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < C / 2; ++w) {
      const float2 k0 = make_float2(bf16_lo(lo[w]), bf16_lo(hi[w]));
      const float2 k1 = make_float2(bf16_hi(lo[w]), bf16_hi(hi[w]));
      a2 = __ffma2_rn(Wc[2 * w], k0, a2);
      a2 = __ffma2_rn(Wc[2 * w + 1], k1, a2);
    }
    acc[i] = a2.x + a2.y;
#pragma unroll
    for (int e = 0; e < C; ++e) {
      const float2 nx = __ffma2_rn(L.twoc[e], Wn[e], make_float2(-Wc[e].x, -Wc[e].y));
      Wc[e] = Wn[e];
      Wn[e] = nx;
    }
  }
  // transposed reduction over the NP lanes of a token phase
  int cnt = TPL;
#pragma unroll
  for (int o = NP / 2; o > 0; o >>= 1) {
    if (cnt > 1) {
      const int half = cnt / 2;
      const bool up = (L.P & o) != 0;
#pragma unroll
      for (int k = 0; k < (TPL > 1 ? TPL / 2 : 1); ++k) {
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
  return acc[0];
}

// Histogram update of one page: H[code][g] += weight of each token.
template <int D, int C>
__device__ inline void page_scatter(const unsigned char* pg, const float* pw, float* Hs, int lane) {
  using X = Dec<D, C>;
  constexpr int NG = X::NG, TPV = X::TPV, VPL = X::VPL;
  const int gv = lane % NG, tp = lane / NG;
  const uint2 wv = *reinterpret_cast<const uint2*>(pg + NG * kPage + gv * kPage);
  if constexpr (TPV == 1) {
    const float4 pa = *reinterpret_cast<const float4*>(pw);
    const float4 pb = *reinterpret_cast<const float4*>(pw + 4);
    const float p[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t code = __byte_perm(t < 4 ? wv.x : wv.y, 0u, 0x4440u | (t & 3));
      atomicAdd(&Hs[code * NG + gv], p[t]);
    }
  } else {
#pragma unroll
    for (int jv = 0; jv < VPL; ++jv) {
      const int t = tp + TPV * jv;
      const uint32_t w = t < 4 ? wv.x : wv.y;
      const uint32_t code = (w >> (8 * (t & 3))) & 0xffu;
      atomicAdd(&Hs[(code * TPV + tp) * NG + gv], pw[t]);
    }
  }
}

template <int D, int C>
__global__ void __launch_bounds__(kThr, 1) decode_kernel(
    Geo g, int layer, int step, const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ ctx_len,
    const int32_t* __restrict__ coded_len, const __nv_bfloat16* __restrict__ sink,
    const __nv_bfloat16* __restrict__ ring, const uint8_t* __restrict__ idx,
    const __nv_bfloat16* __restrict__ cbp, const float* __restrict__ rope, int ns,
    float* __restrict__ ws, float* __restrict__ out, float* __restrict__ lse, float* __restrict__ split_lse,
    int32_t* st) {
  using X = Dec<D, C>;
  constexpr int F = X::F, NG = X::NG, TQ = X::TQ, GRP = X::GRP;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* Ks = smem;
  float* Hs = reinterpret_cast<float*>(smem + X::OFF_H);
  unsigned char* ringb = smem + X::OFF_RING;
  float* sc = reinterpret_cast<float*>(smem + X::OFF_SC);
  float* pwall = reinterpret_cast<float*>(smem + X::OFF_PW);
  float2* zq = reinterpret_cast<float2*>(smem + X::OFF_ZQ);
  float* red = reinterpret_cast<float*>(smem + X::OFF_RED);
  int* misc = reinterpret_cast<int*>(smem + X::OFF_MISC);        // [0]: guard flags, [1]: merge flag
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);
  // bars[0]: key slice (or the bf16 tokens); bars[1 + s]: stage s full; bars[1 + kStages + s]: stage s empty

  const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int h = hq / (g.Hq / g.H);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == kCW;
  const int blk = step / g.Tc, s = step % g.Tc;
  const size_t slot_base = ((size_t)b * g.Hq + hq) * (g.max_splits + 1);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + (size_t)g.B * g.Hq * (g.max_splits + 1) * (D + 2));

  const int ctx = ctx_len[b], Lc = coded_len[b];
  const int S_eff = min(g.S, max(ctx, 0));
  const int recent = ctx - S_eff - Lc;
  const bool bad = ctx < 1 || ctx > g.max_ctx || Lc < 0 || Lc > g.P * kPage ||
                   (Lc > 0 && ctx < g.S + Lc) || recent < 0 || recent > g.R;
  if (bad && j == 0 && tid == 0) set_status(st, LVQ_ECAPACITY);

  int chunk = (Lc + ns - 1) / ns;
  chunk = (chunk + 31) & ~31;
  const int n0 = (bad || j >= ns) ? 0 : min(Lc, j * chunk);
  const int n1 = (bad || j >= ns) ? 0 : min(Lc, n0 + chunk);
  const bool do_coded = n0 < n1;
  const int n_chunks = do_coded ? (n1 - n0 + kChunk - 1) / kChunk : 0;
  const uint8_t* pages = idx + idx_page_off(g, layer, blk, b, h, 0);

  if (tid == 0) {
    mbar_init(smem_addr(&bars[0]), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_addr(&bars[1 + i]), 1);
      mbar_init(smem_addr(&bars[1 + kStages + i]), kCW);
    }
    fence_mbar_init();
    misc[0] = 0;
    misc[1] = 0;
  }
  // query rotated at its own position, scaled so scores come out in log2 units
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
  if (j < ns)
    for (int i = tid; i < X::HF; i += blockDim.x) Hs[i] = 0.f;
  __syncthreads();

  float m_ref = -INFINITY, l_acc = 0.f, m_run = -INFINITY;
  bool timed_out = false;
  if (do_coded) {
    if (producer) {
      // ---- producer warp: the key slice, then the chunks through the ring
      if (lane == 0) {
        const uint32_t bar0 = smem_addr(&bars[0]);
        mbar_expect_tx(bar0, X::KS);
        bulk_g2s(smem_addr(Ks), cbp + cbp_slice_off(g, layer, 0, blk, h, s), X::KS, bar0);
        for (int ci = 0; ci < n_chunks; ++ci) {
          if (ci >= kStages &&
              !mbar_wait(smem_addr(&bars[1 + kStages + ci % kStages]), (ci / kStages - 1) & 1, kWaitIters)) {
            timed_out = true;
            break;
          }
          const int c0 = n0 + ci * kChunk;
          const int np = (min(n1, c0 + kChunk) - c0 + kPage - 1) / kPage;
          const uint32_t bar = smem_addr(&bars[1 + ci % kStages]);
          mbar_expect_tx(bar, np * X::PAGE);
          bulk_g2s(smem_addr(ringb + (ci % kStages) * X::STAGE), pages + (size_t)(c0 / kPage) * X::PAGE,
                   np * X::PAGE, bar);
        }
      }
    } else {
      // ---- compute warps
      Lane<D, C> L;
      lane_init<D, C>(L, lane, zq, rope, g.RC);
      float2 echunk[C], U[C];
      const int p_first = g.S + n0 + kPage * kPPW * warp + L.tq;
#pragma unroll
      for (int e = 0; e < C; ++e) {
        const int f = L.P * C + e;
        echunk[e] = cconj(rope_at(rope, g.RC, F, kChunk, f));
        U[e] = cmul(L.z[e], cconj(rope_at(rope, g.RC, F, p_first, f)));
      }
      float* pw = pwall + warp * kPage;
      const bool writer = (L.P % GRP) == 0;
      const int t_own = L.tq + TQ * (L.P / GRP);
      // waits are bounded and their outcome is made uniform over the warp
      timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[0]), 0, kWaitIters));
      if (!timed_out) timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[1]), 0, kWaitIters));

      // reference maximum: the largest score of every warp's first page.  Every
      // compute warp reaches this barrier exactly once, timed out or not.
      float2 Wc[C], Wn[C];
#pragma unroll
      for (int e = 0; e < C; ++e) { Wc[e] = U[e]; Wn[e] = cmul(U[e], L.etq[e]); }
      const int tb0 = n0 + kPage * (warp * kPPW);
      float sc0 = -INFINITY;
      if (!timed_out && tb0 < n1) sc0 = page_scores<D, C>(L, Ks, ringb + (warp * kPPW) * X::PAGE, Wc, Wn);
      {
        const float wm = warp_max(tb0 + t_own < n1 ? sc0 : -INFINITY);
        if (lane == 0) red[warp] = wm;
        compute_sync();
        m_ref = red[0];
        for (int w = 1; w < kCW; ++w) m_ref = fmaxf(m_ref, red[w]);
      }

      for (int ci = 0; ci < n_chunks && !timed_out; ++ci) {
        const int c0 = n0 + ci * kChunk;
        if (ci > 0) {
          timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[1 + ci % kStages]), (ci / kStages) & 1,
                                                         kWaitIters));
          if (timed_out) break;
#pragma unroll
          for (int e = 0; e < C; ++e) { Wc[e] = U[e]; Wn[e] = cmul(U[e], L.etq[e]); }
        }
        const unsigned char* stage = ringb + (ci % kStages) * X::STAGE;
#pragma unroll 1
        for (int pi = 0; pi < kPPW; ++pi) {
          const int pl = warp * kPPW + pi;
          const int tb = c0 + kPage * pl;
          if (tb >= n1) break;
          const float sc_own = (ci == 0 && pi == 0) ? sc0 : page_scores<D, C>(L, Ks, stage + pl * X::PAGE, Wc, Wn);
          const bool valid = tb + t_own < n1;
          const float sv = valid ? sc_own : -INFINITY;
          m_run = fmaxf(m_run, sv);
          if (sv - m_ref > kGuardLog2) atomicOr(&misc[0], 1);
          const float p = valid ? exp2f(fminf(sv - m_ref, kGuardLog2)) : 0.f;
          if (writer) {
            pw[t_own] = p;
            l_acc += p;
          }
          __syncwarp();
          page_scatter<D, C>(stage + pl * X::PAGE, pw, Hs, lane);
          __syncwarp();
        }
        if (lane == 0) mbar_arrive(smem_addr(&bars[1 + kStages + ci % kStages]));
#pragma unroll
        for (int e = 0; e < C; ++e) U[e] = cmul(U[e], echunk[e]);
      }
    }
  }
  if (__syncthreads_or(timed_out)) {
    if (tid == 0) {
      set_status(st, LVQ_ETIMEOUT);
      misc[0] |= 2;
    }
    // let every issued copy land before the CTA can exit
    if (tid == 0 && do_coded) {
      mbar_wait(smem_addr(&bars[0]), 0, kWaitIters);
      for (int ci = 0; ci < min(n_chunks, kStages); ++ci)
        mbar_wait(smem_addr(&bars[1 + ci]), 0, kWaitIters);
    }
    __syncthreads();
  }

  // ---- rare exact fallback: a score beyond m_ref + 2^64 -> recompute with the true maximum
  if (do_coded && misc[0] == 1) {
    const float m_true = block_reduce<true>(m_run, red);
    for (int i = tid; i < X::HF; i += blockDim.x) Hs[i] = 0.f;
    __syncthreads();
    m_ref = m_true;
    l_acc = 0.f;
    if (!producer) {
      Lane<D, C> L;
      lane_init<D, C>(L, lane, zq, rope, g.RC);
      float* pw = pwall + warp * kPage;
      const bool writer = (L.P % GRP) == 0;
      const int t_own = L.tq + TQ * (L.P / GRP);
      for (int tb = n0 + kPage * warp; tb < n1; tb += kPage * kCW) {
        const unsigned char* pg = pages + (size_t)(tb / kPage) * X::PAGE;   // straight from global memory
        float2 Wc[C], Wn[C];
#pragma unroll
        for (int e = 0; e < C; ++e) {
          Wc[e] = cmul(L.z[e], cconj(rope_at(rope, g.RC, F, g.S + tb + L.tq, L.P * C + e)));
          Wn[e] = cmul(Wc[e], L.etq[e]);
        }
        const float sc_own = page_scores<D, C>(L, Ks, pg, Wc, Wn);
        const bool valid = tb + t_own < n1;
        const float p = valid ? exp2f(sc_own - m_ref) : 0.f;
        if (writer) {
          pw[t_own] = p;
          l_acc += p;
        }
        __syncwarp();
        page_scatter<D, C>(pg, pw, Hs, lane);
        __syncwarp();
      }
    }
    __syncthreads();
  }

  // ---- coded partial: o[e] = sum_k H[k][g] V[k][g][e mod c]
  if (j < ns) {
    float* part = ws + (slot_base + j) * (D + 2);
    const float l_tot = block_reduce<false>(producer ? 0.f : l_acc, red);
    constexpr int NKQ = kCT / D;
    float o = 0.f;
    if (do_coded && !producer) {
      const int e = tid % D, kq = tid / D, grp = e / C, ee = e % C;
      const __nv_bfloat16* Vs = cbp + cbp_slice_off(g, layer, 1, blk, h, s) + (size_t)grp * C + ee;
#pragma unroll 8
      for (int k = kq; k < kEntries; k += NKQ) {
        float hsum = 0.f;
#pragma unroll
        for (int t2 = 0; t2 < X::TPV; ++t2) hsum += Hs[(k * X::TPV + t2) * NG + grp];
        o = fmaf(hsum, __bfloat162float(Vs[(size_t)k * D]), o);
      }
    }
    __syncthreads();
    if (!producer) Hs[tid] = o;      // Hs holds kCT partial sums now
    __syncthreads();
    if (tid < D) {
      float oe = 0.f;
#pragma unroll
      for (int k2 = 0; k2 < NKQ; ++k2) oe += Hs[k2 * D + tid];
      part[tid] = oe;
    }
    if (tid == 0) {
      const bool ok = do_coded && !(misc[0] & 2);
      part[D] = ok ? m_ref : -INFINITY;
      part[D + 1] = ok ? l_tot : 0.f;
    }
  }

  // ---- CTA ns: the bf16 partial (sink tokens and recent window)
  if (j == ns) {
    float* pb = ws + (slot_base + ns) * (D + 2);
    const int nb = bad ? 0 : S_eff + recent;
    __nv_bfloat16* Kb = reinterpret_cast<__nv_bfloat16*>(smem);                 // [S + R][D]
    __nv_bfloat16* Vb = Kb + (size_t)(g.S + g.R) * D;                            // [S + R][D]
    bool ok = true;
    if (nb > 0) {
      const uint32_t barb = smem_addr(&bars[0]);
      if (tid == 0) {
        const uint32_t sb = (uint32_t)S_eff * D * 2, rb = (uint32_t)g.R * D * 2;
        mbar_expect_tx(barb, 2 * (sb + rb));
        if (sb) {
          bulk_g2s(smem_addr(Kb), sink + sink_off(g, layer, 0, step, b, h, 0), sb, barb);
          bulk_g2s(smem_addr(Vb), sink + sink_off(g, layer, 1, step, b, h, 0), sb, barb);
        }
        bulk_g2s(smem_addr(Kb + (size_t)g.S * D), ring + ring_off(g, layer, 0, step, b, h, 0), rb, barb);
        bulk_g2s(smem_addr(Vb + (size_t)g.S * D), ring + ring_off(g, layer, 1, step, b, h, 0), rb, barb);
      }
      ok = !__syncthreads_or(!mbar_wait(barb, 0, kWaitIters));
      if (!ok && tid == 0) set_status(st, LVQ_ETIMEOUT);
    }
    // scores: 4 threads per token, each a quarter of the frequencies
    constexpr int FQ = F / 4;
    for (int i0 = 0; i0 < nb && ok; i0 += kCT / 4) {
      const int i = i0 + tid / 4, qf = tid % 4;
      float part_s = 0.f;
      if (i < nb && tid < kCT) {
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
      if (i < nb && qf == 0 && tid < kCT) sc[i] = part_s;
    }
    __syncthreads();
    float mloc = -INFINITY;
    for (int i = tid; i < nb && ok; i += blockDim.x) mloc = fmaxf(mloc, sc[i]);
    const float M = block_reduce<true>(mloc, red);
    float lloc = 0.f;
    for (int i = tid; i < nb && ok; i += blockDim.x) {
      const float p = exp2f(sc[i] - M);
      sc[i] = p;
      lloc += p;
    }
    const float Lb = block_reduce<false>(lloc, red);     // block_reduce syncs: sc holds the weights
    constexpr int NTS = kCT / D;
    float o = 0.f;
    if (tid < kCT) {
      const int e = tid % D, ts = tid / D;
      for (int i = ts; i < nb && ok; i += NTS) {
        const int row = i < S_eff ? i : g.S + (Lc + (i - S_eff)) % g.R;
        o = fmaf(sc[i], __bfloat162float(Vb[(size_t)row * D + e]), o);
      }
    }
    __syncthreads();
    if (tid < kCT) Hs[tid] = o;    // after the barrier nothing reads the staged tokens any more
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
  if (tid == 0) misc[1] = atomicAdd(&counters[(size_t)b * g.Hq + hq], 1) == ns;
  __syncthreads();
  if (!misc[1]) return;
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
  decode_kernel<D, C><<<grid, kThr, Dec<D, C>::SMEM, s>>>(g, layer, step, q, ctx_len, coded_len, sink, ring, idx,
                                                          cbp, rope, ns, ws, out, lse, split_lse, st);
  return cudaGetLastError();
}

// bf16 tokens (sink + ring slots) the bf16-partial CTA can stage: K and V must
// fit below the score buffer, and their scores in it.
template <int D, int C>
static int bf16_capacity_as() {
  const int by_smem = Dec<D, C>::OFF_SC / (4 * D);
  return by_smem < Dec<D, C>::SC_N ? by_smem : Dec<D, C>::SC_N;
}

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
