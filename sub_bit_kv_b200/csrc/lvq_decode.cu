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
//  * Coded split j < num_splits: the producer bulk-copies the step-t key and
//    value slices of the head's codebooks ([256][n_g][c] bf16 each, one
//    contiguous span each) and then the split's code pages, 480 tokens per
//    chunk, through a 3-stage ring (cp.async.bulk into shared memory, no
//    multicast; full/empty mbarriers).  Each compute warp takes 4 consecutive
//    pages of every chunk.
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
//  * Values: lane (tp, g) owns group g's c channels and accumulates
//    p * V_slice[code][g] for every (32/n_g)-th token in fp32 registers, with
//    an online softmax per warp (the warp's reference maximum is raised, and
//    its accumulators rescaled, only when a score exceeds it by 2^16).
//  * CTA num_splits computes the bf16 tokens' partial (sink and recent window)
//    from shared-memory copies of the tokens and of the RoPE table rows.
//  * The last CTA of a (request, head) to finish merges the partials by LSE
//    (a counter in the workspace, returned to zero by that CTA).
#include "lvq_common.cuh"

namespace lvq {

constexpr int kCW = 15;                      // compute warps (+1 producer: 512 threads, 128 registers)
constexpr int kCT = 32 * kCW;                // compute threads
constexpr int kThr = kCT + 32;
constexpr int kPPW = 4;                      // pages per warp per chunk
constexpr int kChunk = kPage * kCW * kPPW;   // 480 coded tokens per chunk
constexpr int kStages = 3;
constexpr float kRaiseLog2 = 16.f;           // raise a warp's reference maximum beyond this margin

template <int D, int C>
struct Dec {
  static constexpr int F = D / 2;          // RoPE frequencies
  static constexpr int NG = D / C;         // groups per step
  static constexpr int NP = NG / 2;        // pair-groups (groups g, g + NG/2)
  static constexpr int TQ = 32 / NP;       // token phases of the score mapping
  static constexpr int TPL = kPage / TQ;   // score tokens per lane per page
  static constexpr int GRP = NP / TPL;     // lanes holding the same reduced score
  static constexpr int TPV = 32 / NG;      // token phases of the value mapping
  static constexpr int VPL = kPage / TPV;   // value tokens per lane per page
  static constexpr int PAGE = 2 * NG * kPage;
  static constexpr int STAGE = (kChunk / kPage) * PAGE;
  static constexpr int KS = kEntries * D * 2;                     // one step slice, K or V
  static constexpr int OFF_V = KS;
  static constexpr int OFF_RING = 2 * KS;
  static constexpr int OFF_PW = OFF_RING + kStages * STAGE;       // per-warp (p, p) pairs of a page
  static constexpr int OFF_ZQ = OFF_PW + kCW * kPage * 8;
  static constexpr int OFF_RED = OFF_ZQ + F * 8;
  static constexpr int OFF_MISC = OFF_RED + 64 * 4;
  static constexpr int OFF_BAR = OFF_MISC + 16;
  static constexpr int SMEM = OFF_BAR + 8 * (2 * kStages + 1) + 8;
  static_assert(NP >= 4 && NP <= 32 && 32 % NP == 0, "pair-group mapping");
  static_assert(NG <= 32 && 32 % NG == 0, "value mapping");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(OFF_RING % 16 == 0 && OFF_PW % 16 == 0, "alignment");
  static_assert(kStages * STAGE >= kCW * (D + 2) * 4, "warp partials fit in the ring");
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

__device__ inline void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

// Address of a slice row: code * (2d) + byte offset of the group.  For d = 128
// the row is 256 bytes, so one byte permute places the code byte in bits 8-15
// and the group offset in bits 0-7.
template <int D>
__device__ inline uint32_t row_addr(uint32_t word, uint32_t gbyte, uint32_t sel) {
  if constexpr (D * 2 == 256) {
    return __byte_perm(word, gbyte, sel);
  } else {
    return (__byte_perm(word, 0u, sel) >> 8) * (D * 2) + gbyte;
  }
}
// selector: byte 0 <- second operand byte 0, byte 1 <- first operand byte bpos, bytes 2-3 <- zero
__device__ inline uint32_t row_sel(int bpos) { return 0x5504u | ((uint32_t)(bpos & 3) << 4); }

template <int C>
__device__ inline void load_row(const unsigned char* base, uint32_t off, uint32_t (&w)[C / 2]) {
  if constexpr (C == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(base + off);
    w[0] = a.x; w[1] = a.y;
  } else {
#pragma unroll
    for (int q = 0; q < C / 8; ++q) {
      const uint4 a = *reinterpret_cast<const uint4*>(base + off + 16 * q);
      w[4 * q + 0] = a.x; w[4 * q + 1] = a.y; w[4 * q + 2] = a.z; w[4 * q + 3] = a.w;
    }
  }
}

// Per-lane state of the score mapping.
template <int D, int C>
struct Lane {
  int P, tq;
  uint32_t gb_lo, gb_hi;              // byte offsets of the lane's two groups inside a slice row
  uint32_t sel[2];
  float2 twoc[C], etq[C];
};

template <int D, int C>
__device__ inline void lane_init(Lane<D, C>& L, int lane, const float* rope, int RC) {
  using X = Dec<D, C>;
  constexpr int NP = X::NP, TQ = X::TQ, F = X::F;
  L.P = lane % NP;
  L.tq = lane / NP;
  L.gb_lo = (uint32_t)L.P * C * 2;
  L.gb_hi = (uint32_t)(L.P + NP) * C * 2;
  L.sel[0] = row_sel(L.tq);
  L.sel[1] = row_sel(L.tq + (TQ == 2 ? 2 : 0));
#pragma unroll
  for (int e = 0; e < C; ++e) {
    const int f = L.P * C + e;
    const float2 r = rope_at(rope, RC, F, TQ, f);
    L.twoc[e] = make_float2(2.f * r.x, 2.f * r.x);
    L.etq[e] = cconj(r);
  }
}

// Scores of the 8 tokens of one page.  On return the lane holds the score of
// token t_own = tq + TQ * (P / GRP); W advances by TPL tokens.
template <int D, int C>
__device__ inline float page_scores(const Lane<D, C>& L, const unsigned char* Ks, const unsigned char* pg,
                                    float2 (&Wc)[C], float2 (&Wn)[C]) {
  using X = Dec<D, C>;
  constexpr int TQ = X::TQ, TPL = X::TPL, NP = X::NP;
  const uint2 wlo = *reinterpret_cast<const uint2*>(pg + L.P * kPage);
  const uint2 whi = *reinterpret_cast<const uint2*>(pg + (L.P + NP) * kPage);
  float acc[TPL];
#pragma unroll
  for (int i = 0; i < TPL; ++i) {
    uint32_t xl, xh, sel;
    if constexpr (TQ == 8) {
      xl = L.tq < 4 ? wlo.x : wlo.y;
      xh = L.tq < 4 ? whi.x : whi.y;
      sel = L.sel[0];
    } else {
      const int word = (TQ * i) / 4;                 // compile-time
      xl = word ? wlo.y : wlo.x;
      xh = word ? whi.y : whi.x;
      sel = L.sel[(TQ * i / 2) & 1];
    }
    uint32_t lo[C / 2], hi[C / 2];
    load_row<C>(Ks, row_addr<D>(xl, L.gb_lo, sel), lo);
    load_row<C>(Ks, row_addr<D>(xh, L.gb_hi, sel), hi);
    float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < C / 2; ++w) {
      a2 = __ffma2_rn(Wc[2 * w], make_float2(bf16_lo(lo[w]), bf16_lo(hi[w])), a2);
      a2 = __ffma2_rn(Wc[2 * w + 1], make_float2(bf16_hi(lo[w]), bf16_hi(hi[w])), a2);
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

// o += p_t * V_slice[code_t][g] over the lane's tokens of one page.
template <int D, int C>
__device__ inline void page_values(const unsigned char* Vsm, const unsigned char* pg, const float2* pw2, int gv,
                                   int tp, uint32_t gbv, float2 (&o)[C / 2]) {
  using X = Dec<D, C>;
  constexpr int NG = X::NG, TPV = X::TPV, VPL = X::VPL;
  const uint2 wv = *reinterpret_cast<const uint2*>(pg + NG * kPage + gv * kPage);
#pragma unroll
  for (int jv = 0; jv < VPL; ++jv) {
    const int t = tp + TPV * jv;
    uint32_t word, sel;
    if constexpr (TPV == 1) {
      word = jv < 4 ? wv.x : wv.y;
      sel = row_sel(jv);
    } else {
      word = t < 4 ? wv.x : wv.y;
      sel = row_sel(t);
    }
    uint32_t v[C / 2];
    load_row<C>(Vsm, row_addr<D>(word, gbv, sel), v);
    const float2 p2 = pw2[t];
#pragma unroll
    for (int w = 0; w < C / 2; ++w) o[w] = __ffma2_rn(p2, make_float2(bf16_lo(v[w]), bf16_hi(v[w])), o[w]);
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
  constexpr int F = X::F, NG = X::NG, TQ = X::TQ, GRP = X::GRP, TPV = X::TPV;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* Ks = smem;
  unsigned char* Vsm = smem + X::OFF_V;
  unsigned char* ringb = smem + X::OFF_RING;
  float2* pwall = reinterpret_cast<float2*>(smem + X::OFF_PW);
  float2* zq = reinterpret_cast<float2*>(smem + X::OFF_ZQ);
  float* red = reinterpret_cast<float*>(smem + X::OFF_RED);
  int* misc = reinterpret_cast<int*>(smem + X::OFF_MISC);        // [0]: failure flag, [1]: merge flag
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);
  // bars[0]: slices (or the bf16 tokens); bars[1 + s]: stage s full; bars[1 + kStages + s]: stage s empty

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
  __syncthreads();

  bool timed_out = false;
  float m_w = -INFINITY, l_w = 0.f;       // warp's reference maximum (log2) and weight sum (writer lanes)
  float2 o[C / 2];
#pragma unroll
  for (int w = 0; w < C / 2; ++w) o[w] = make_float2(0.f, 0.f);

  if (do_coded) {
    if (producer) {
      // ---- producer: the two step slices, then the chunks through the ring
      if (lane == 0) {
        const uint32_t bar0 = smem_addr(&bars[0]);
        mbar_expect_tx(bar0, 2 * X::KS);
        bulk_g2s(smem_addr(Ks), cbp + cbp_slice_off(g, layer, 0, blk, h, s), X::KS, bar0);
        bulk_g2s(smem_addr(Vsm), cbp + cbp_slice_off(g, layer, 1, blk, h, s), X::KS, bar0);
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
      lane_init<D, C>(L, lane, rope, g.RC);
      float2 echunk[C], U[C];
      const int p_first = g.S + n0 + kPage * kPPW * warp + L.tq;
#pragma unroll
      for (int e = 0; e < C; ++e) {
        const int f = L.P * C + e;
        echunk[e] = cconj(rope_at(rope, g.RC, F, kChunk, f));
        U[e] = cmul(zq[f], cconj(rope_at(rope, g.RC, F, p_first, f)));
      }
      float2* pw2 = pwall + warp * kPage;
      const bool writer = (L.P % GRP) == 0;
      const int t_own = L.tq + TQ * (L.P / GRP);
      const int gv = lane % NG, tp = lane / NG;
      const uint32_t gbv = (uint32_t)gv * C * 2;
      // waits are bounded; their outcome is made uniform over the warp
      timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[0]), 0, kWaitIters));

      for (int ci = 0; ci < n_chunks && !timed_out; ++ci) {
        const int c0 = n0 + ci * kChunk;
        timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[1 + ci % kStages]), (ci / kStages) & 1,
                                                       kWaitIters));
        if (timed_out) break;
        const unsigned char* stage = ringb + (ci % kStages) * X::STAGE;
        float2 Wc[C], Wn[C];
#pragma unroll
        for (int e = 0; e < C; ++e) { Wc[e] = U[e]; Wn[e] = cmul(U[e], L.etq[e]); }
#pragma unroll 1
        for (int pi = 0; pi < kPPW; ++pi) {
          const int pl = warp * kPPW + pi;
          const int tb = c0 + kPage * pl;
          if (tb >= n1) break;
          const unsigned char* pg = stage + pl * X::PAGE;
          const float sc = page_scores<D, C>(L, Ks, pg, Wc, Wn);
          const bool valid = tb + t_own < n1;
          const float sv = valid ? sc : -INFINITY;
          // online softmax per warp: raise the reference only when a score passes it by 2^16
          if (__any_sync(0xffffffffu, sv > m_w + kRaiseLog2)) {
            const float m_new = fmaxf(m_w, warp_max(sv));
            const float alpha = exp2f(m_w - m_new);     // 0 for the first page
#pragma unroll
            for (int w = 0; w < C / 2; ++w) o[w] = make_float2(o[w].x * alpha, o[w].y * alpha);
            l_w *= alpha;
            m_w = m_new;
          }
          const float p = valid ? exp2f(sv - m_w) : 0.f;
          if (writer) {
            pw2[t_own] = make_float2(p, p);
            l_w += p;
          }
          __syncwarp();
          page_values<D, C>(Vsm, pg, pw2, gv, tp, gbv, o);
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
      misc[0] = 1;
      if (do_coded) {   // let every issued copy land before the CTA can exit
        mbar_wait(smem_addr(&bars[0]), 0, kWaitIters);
        for (int ci = 0; ci < min(n_chunks, kStages); ++ci) mbar_wait(smem_addr(&bars[1 + ci]), 0, kWaitIters);
      }
    }
    __syncthreads();
  }

  // ---- coded partial: combine the warps' (m, l, o) -- staged in the free ring
  if (j < ns) {
    float* part = ws + (slot_base + j) * (D + 2);
    float* wo = reinterpret_cast<float*>(ringb);          // [kCW][D + 2]
    if (!producer) {
      // sum the value accumulators over the lanes sharing a group
#pragma unroll
      for (int off = NG; off < 32; off <<= 1)
#pragma unroll
        for (int w = 0; w < C / 2; ++w) {
          o[w].x += __shfl_xor_sync(0xffffffffu, o[w].x, off);
          o[w].y += __shfl_xor_sync(0xffffffffu, o[w].y, off);
        }
      const float lsum = warp_sum(l_w);
      float* mine = wo + warp * (D + 2);
      if (lane < NG) {
#pragma unroll
        for (int w = 0; w < C / 2; ++w) {
          mine[lane * C + 2 * w] = o[w].x;
          mine[lane * C + 2 * w + 1] = o[w].y;
        }
      }
      if (lane == 0) { mine[D] = m_w; mine[D + 1] = lsum; }
    }
    __syncthreads();
    const bool ok = do_coded && !misc[0];
    float M = -INFINITY;
    for (int w = 0; w < kCW; ++w) M = fmaxf(M, wo[w * (D + 2) + D]);
    if (tid < D) {
      float oe = 0.f;
      if (ok && M != -INFINITY)
        for (int w = 0; w < kCW; ++w) {
          const float mw = wo[w * (D + 2) + D];
          if (mw != -INFINITY) oe = fmaf(exp2f(mw - M), wo[w * (D + 2) + tid], oe);
        }
      part[tid] = oe;
    }
    if (tid == 0) {
      float Ls = 0.f;
      if (ok && M != -INFINITY)
        for (int w = 0; w < kCW; ++w) {
          const float mw = wo[w * (D + 2) + D];
          if (mw != -INFINITY) Ls = fmaf(exp2f(mw - M), wo[w * (D + 2) + D + 1], Ls);
        }
      part[D] = ok ? M : -INFINITY;
      part[D + 1] = ok ? Ls : 0.f;
    }
  }

  // ---- CTA ns: the bf16 partial (sink tokens and recent window)
  if (j == ns) {
    float* pb = ws + (slot_base + ns) * (D + 2);
    const int nb = bad ? 0 : S_eff + recent;
    const int nrow = g.S + g.R;
    __nv_bfloat16* Kb = reinterpret_cast<__nv_bfloat16*>(smem);          // [S + R][D]
    __nv_bfloat16* Vb = Kb + (size_t)nrow * D;                             // [S + R][D]
    // RoPE rows: sink positions [0, S) use coarse rows 0..; recent positions use coarse rows r0..r1
    float2* fine_s = reinterpret_cast<float2*>(Vb + (size_t)nrow * D);    // [8][F]
    float2* coarse_s = fine_s + 8 * F;                                     // [n_sink_rows + n_rec_rows][F]
    float* sc = reinterpret_cast<float*>(coarse_s);                        // reused after the scores
    const int sink_rows = (S_eff + 7) / 8;
    const int r0 = (g.S + Lc) >> 3, r1 = recent > 0 ? (ctx - 1) >> 3 : r0 - 1;
    const int rec_rows = r1 - r0 + 1;
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
      const float2* rp = reinterpret_cast<const float2*>(rope);
      for (int i = tid; i < 8 * F; i += blockDim.x) fine_s[i] = rp[(size_t)g.RC * F + i];
      for (int i = tid; i < sink_rows * F; i += blockDim.x) coarse_s[i] = rp[i];
      for (int i = tid; i < rec_rows * F; i += blockDim.x) coarse_s[sink_rows * F + i] = rp[(size_t)r0 * F + i];
      ok = !__syncthreads_or(!mbar_wait(barb, 0, kWaitIters));
      if (!ok && tid == 0) set_status(st, LVQ_ETIMEOUT);
    }
    // scores: 4 threads per token, a quarter of the frequencies each
    constexpr int FQ = F / 4;
    float my_sc[4];
    int n_mine = 0;
    for (int i0 = 0; i0 < nb && ok; i0 += kThr / 4) {
      const int i = i0 + tid / 4, qf = tid % 4;
      float part_s = 0.f;
      if (i < nb) {
        int pos, row, crow;
        if (i < S_eff) { pos = i; row = i; crow = pos >> 3; }
        else {
          pos = g.S + Lc + (i - S_eff);
          row = g.S + (pos - g.S) % g.R;
          crow = sink_rows + (pos >> 3) - r0;
        }
        const __nv_bfloat16* kr = Kb + (size_t)row * D;
        const float2* cr = coarse_s + (size_t)crow * F;
        const float2* fr = fine_s + (size_t)(pos & 7) * F;
#pragma unroll 4
        for (int f = qf * FQ; f < (qf + 1) * FQ; ++f) {
          const float2 w = cmul(zq[f], cconj(cmul(cr[f], fr[f])));
          part_s = fmaf(w.x, __bfloat162float(kr[f]), part_s);
          part_s = fmaf(w.y, __bfloat162float(kr[f + F]), part_s);
        }
      }
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 1);
      part_s += __shfl_xor_sync(0xffffffffu, part_s, 2);
      my_sc[n_mine++ & 3] = part_s;           // the thread's tokens i0/4-stride (at most 4 passes)
    }
    // maximum and weights (each token's score lives in its 4 threads)
    float mloc = -INFINITY;
    for (int k = 0, i0 = 0; i0 < nb && ok; i0 += kThr / 4, ++k)
      if (i0 + tid / 4 < nb) mloc = fmaxf(mloc, my_sc[k & 3]);
    const float M = block_reduce<true>(mloc, red);
    __syncthreads();                           // the RoPE rows are no longer read: sc may overwrite them
    float lloc = 0.f;
    for (int k = 0, i0 = 0; i0 < nb && ok; i0 += kThr / 4, ++k) {
      const int i = i0 + tid / 4;
      if (i < nb && (tid % 4) == 0) {
        const float p = exp2f(my_sc[k & 3] - M);
        sc[i] = p;
        lloc += p;
      }
    }
    const float Lb = block_reduce<false>(lloc, red);     // block_reduce syncs: sc holds the weights
    constexpr int NTS = kThr / D;
    float ov = 0.f;
    {
      const int e = tid % D, ts = tid / D;
      for (int i = ts; i < nb && ok; i += NTS) {
        const int row = i < S_eff ? i : g.S + (Lc + (i - S_eff)) % g.R;
        ov = fmaf(sc[i], __bfloat162float(Vb[(size_t)row * D + e]), ov);
      }
    }
    __syncthreads();
    float* parts = reinterpret_cast<float*>(smem);      // the staged tokens are no longer read
    parts[tid] = ov;
    __syncthreads();
    if (tid < D) {
      float oe = 0.f;
#pragma unroll
      for (int k2 = 0; k2 < NTS; ++k2) oe += parts[k2 * D + tid];
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
  float* lse2 = red + 32;                     // up to 32 partials via red[], else recomputed below
  (void)lse2;
  float M = -INFINITY;
  for (int i = 0; i <= ns; ++i) {
    const float* pj = base + (size_t)i * (D + 2);
    const float l = __ldcg(pj + D + 1);
    if (l > 0.f) M = fmaxf(M, __ldcg(pj + D) + log2f(l));
  }
  float den = 0.f;
  if (M != -INFINITY)
    for (int i = 0; i <= ns; ++i) {
      const float* pj = base + (size_t)i * (D + 2);
      const float l = __ldcg(pj + D + 1);
      if (l > 0.f) den += exp2f(__ldcg(pj + D) + log2f(l) - M);
    }
  const float L2 = M == -INFINITY ? -INFINITY : M + log2f(den);
  if (tid < D) {
    float ov = 0.f;
    if (M != -INFINITY)
      for (int i = 0; i <= ns; ++i) {
        const float* pj = base + (size_t)i * (D + 2);
        if (__ldcg(pj + D + 1) > 0.f) ov = fmaf(exp2f(__ldcg(pj + D) - L2), __ldcg(pj + tid), ov);
      }
    out[((size_t)b * g.Hq + hq) * D + tid] = ov;
  }
  constexpr float kLn2 = 0.6931471805599453f;
  if (tid == 0) {
    lse[(size_t)b * g.Hq + hq] = L2 * kLn2;
    counters[(size_t)b * g.Hq + hq] = 0;
  }
  if (split_lse)
    for (int i = tid; i <= ns; i += blockDim.x) {
      const float* pj = base + (size_t)i * (D + 2);
      const float l = __ldcg(pj + D + 1);
      split_lse[((size_t)b * g.Hq + hq) * (ns + 1) + i] = l > 0.f ? (__ldcg(pj + D) + log2f(l)) * kLn2 : -INFINITY;
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

// Sink + recent-window slots the bf16-partial CTA can stage: K and V rows, the
// fine RoPE rows and the coarse rows its positions need must fit in its
// shared memory, and its 4-thread-per-token scoring covers at most 4 passes.
template <int D, int C>
static int bf16_capacity_as() {
  const int F = D / 2;
  // bytes: 4*D per token (K and V), 8*F*8 fine rows, (tokens/8 + 3) coarse rows of 8*F
  const int avail = Dec<D, C>::OFF_PW - 8 * F * 8 - 3 * 8 * F;
  const int by_smem = avail / (4 * D + F);
  const int by_passes = 4 * (kThr / 4);
  return by_smem < by_passes ? by_smem : by_passes;
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
