// Split-K decode attention over the LoopVQ coded cache, with the LSE merge
// fused into the same launch.
//
// "LoopVQ summary", section "premises and limits": the attention kernel reads
// only the step-t slice of each codebook, splits the quantized tokens as in
// Flash-Decoding and merges them, and the bf16 sink/recent tokens, by
// logsumexp.  Section "how it differs": keys are stored before RoPE and RoPE is
// applied to the reconstructed key.
//
// Work items (request, query head, split j); 15 compute warps and one producer warp per CTA,
// one CTA per SM.  Item j owns coded split j and every num_splits-th bf16 token (sink and
// recent window), and writes two partials (m, l, o): its coded split and its share of the bf16
// tokens.  Two kernels share the per-item machinery:
//  * decode_kernel: one CTA per item, grid (num_splits, query heads, requests).  The producer
//    warp computes the item's bf16 share (its rows staged through the value-slice area) while
//    the compute warps score the coded split; the value slice is copied after it.
//  * decode_runs_kernel: one CTA per SM, each walking a contiguous, cost-balanced run of items
//    ordered by KV head, so that the step slices of a KV head are copied once per run, the code
//    pages of its query heads are read again from L2, and the producer streams the next item's
//    code pages while the compute warps finish the current one.  The compute warps compute each
//    item's bf16 share straight from global memory.
//  * Coded split: the producer bulk-copies the step-t key slice ([256][n_g][c]
//    bf16, one contiguous span), the value slice, and the split's code pages in
//    480-token chunks through a 3-stage ring (cp.async.bulk, no multicast;
//    full/empty mbarriers): the K pages of a super-chunk, then its V pages.
//  * Phase A (scores): lane (tq, P) of a compute warp owns pair-group P --
//    groups P and P + n_g/2, i.e. the RoPE frequencies f = P*c + e whose
//    rotate-half partners are channels f and f + d/2 -- and every
//    (32/n_p)-th token of the warp's pages.  With z_f = q'_f + i q'_{f+d/2}
//    (the query rotated at its own position), a key k at position p scores
//      sum_f Re(z_f e^{-i p theta_f}) k_f + Im(z_f e^{-i p theta_f}) k_{f+d/2}
//    = q' . RoPE(k, p).  Along a lane's tokens (stride s) the factor
//    W_n = z e^{-i p_n theta} obeys W_{n+1} = 2 cos(s theta) W_n - W_{n-1}: one
//    packed f32x2 FMA per frequency for the rotation and one for the dot
//    product; the recurrence is reseeded exactly at every chunk.  A code byte
//    becomes its shared-memory row address in one byte permute.  Scores go to
//    shared memory.
//  * Between the phases: the exact maximum M of the super-chunk and
//    S = sum 2^(s - M); every weight becomes the integer round(2^(s-M) * 2^k)
//    with 2^k * S < 2^30, so that any sum of weights fits 31 bits and each
//    weight is exact to 2^-31 of S.
//  * Phase B (values): out = sum_t w_t V[code_t] = sum_(a, g) H[a][g] V[a][g],
//    with H[a][g] the sum of the weights of the tokens whose group-g code is
//    a.  Lane g adds its tokens' weights to H with 32-bit shared-memory
//    atomics (integer adds: exact and order-independent; row a of H is 4*n_g
//    bytes, so the 32 lanes of a warp hit 32 distinct banks).  One pass over
//    the value slice then contracts H into o.
//  * The last item of a (request, head) to finish merges the 2 * num_splits
//    partials by LSE (a counter in the workspace, returned to zero by the
//    merging CTA).
#include <type_traits>

#include "lvq_common.cuh"

namespace lvq {

constexpr int kCW = 15;                      // compute warps (+1 producer: 512 threads, 128 registers)
constexpr int kCT = 32 * kCW;                // compute threads
constexpr int kThr = kCT + 32;
constexpr int kPPW = 4;                      // pages per warp per chunk
constexpr int kChunk = kPage * kCW * kPPW;   // 480 coded tokens per chunk
constexpr int kStages = 3;
constexpr int kSmemMax = 227 * 1024;
constexpr int kBarCompute = 1;               // named barrier of the 15 compute warps
constexpr int kMaxSuperChunks = 16;          // chunks per super-chunk, at most

template <int D, int C>
struct Dec {
  static constexpr int F = D / 2;          // RoPE frequencies
  static constexpr int NG = D / C;         // groups per step
  static constexpr int NP = NG / 2;        // pair-groups (groups g, g + NG/2)
  static constexpr int LS = C > 4 ? C / 4 : 1;   // score lanes per pair-group (4 frequencies each)
  static constexpr int CL = C / LS;        // frequencies of one score lane
  static constexpr int NPV = NP * LS;      // score lanes of one token phase
  static constexpr int TQ = 32 / NPV;      // token phases of the score mapping
  static constexpr int TPL = kPage / TQ;   // score tokens per lane per page
  static constexpr int TPV = 32 / NG;      // lanes per group in the value phase
  static constexpr int VPL = kPage / TPV;  // value tokens per lane per page
  static constexpr int SH = NG == 32 ? 7 : NG == 16 ? 6 : 5;   // log2 of a histogram row in bytes
  static constexpr int PAGE = NG * kPage;  // bytes of one K (or V) page
  static constexpr int STAGE = (kChunk / kPage) * PAGE;
  static constexpr int KS = kEntries * D * 2;                     // one step slice, K or V
  static constexpr int HB = kEntries * NG * 4;                    // histogram [256][n_g] u32
  static constexpr int NPAIR = D / 2;                             // channel pairs of the contraction
  static constexpr int NREP = kCT / NPAIR;                        // entry phases of the contraction
  static constexpr int OFF_V = KS;
  static constexpr int OFF_H = 2 * KS;
  static constexpr int OFF_RING = OFF_H + HB;
  static constexpr int OFF_ZQ = OFF_RING + kStages * STAGE;
  static constexpr int OFF_TAB = OFF_ZQ + F * 8;                  // e^{-i TQ theta_f}, e^{-i 480 theta_f}
  static constexpr int OFF_RED = OFF_TAB + 2 * F * 8;
  static constexpr int OFF_MISC = OFF_RED + 64 * 4;
  static constexpr int OFF_BAR = OFF_MISC + 32;
  static constexpr int NBAR = 3 + 2 * kStages;
  static constexpr int OFF_SC = OFF_BAR + (NBAR * 8 + 15) / 16 * 16;
  static constexpr int NSC_FIT = (kSmemMax - OFF_SC) / 4 / kChunk;
  static constexpr int NSC = (NSC_FIT < kMaxSuperChunks ? NSC_FIT : kMaxSuperChunks) * kChunk;
  static constexpr int SMEM = OFF_SC + NSC * 4;
  static_assert(NPV >= 4 && NPV <= 32 && 32 % NPV == 0, "pair-group mapping");
  static_assert(NG >= 8 && NG <= 32 && 32 % NG == 0, "value mapping");
  static_assert((1 << SH) == NG * 4, "histogram row");
  static_assert(NSC >= kChunk && SMEM <= kSmemMax, "shared memory");
  static_assert(NSC >= 3 * 512 && NSC * 4 >= NREP * NPAIR * 8, "scratch in the score array");

  static_assert(OFF_RING % 16 == 0 && OFF_SC % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
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
  int vp, P, tq, f0;                  // lane in its token phase, pair-group, token phase, first frequency
  uint32_t gb_lo, gb_hi;              // byte offsets of the lane's share of its two groups in a slice row
  uint32_t sel[2];
  float2 twoc[Dec<D, C>::CL], mtwoc[Dec<D, C>::CL];   // (2 cos, 2 cos) and its negation, token stride
};

// The score lane `lane` of a token phase covers frequencies [f0, f0 + CL): those of pair-group
// P = vp / LS, share vp % LS.
template <int D, int C>
__device__ inline int lane_f0(int lane) {
  using X = Dec<D, C>;
  const int vp = lane % X::NPV;
  return (vp / X::LS) * C + (vp % X::LS) * X::CL;
}

template <int D, int C>
__device__ inline void lane_init(Lane<D, C>& L, int lane, const float2* etq_s) {
  using X = Dec<D, C>;
  constexpr int NP = X::NP, TQ = X::TQ, CL = X::CL;
  L.vp = lane % X::NPV;
  L.P = L.vp / X::LS;
  L.tq = lane / X::NPV;
  L.f0 = lane_f0<D, C>(lane);
  const uint32_t share = (uint32_t)(L.vp % X::LS) * CL * 2;
  L.gb_lo = (uint32_t)L.P * C * 2 + share;
  L.gb_hi = (uint32_t)(L.P + NP) * C * 2 + share;
  L.sel[0] = row_sel(L.tq);
  L.sel[1] = row_sel(L.tq + (TQ == 2 ? 2 : 0));
#pragma unroll
  for (int e = 0; e < CL; ++e) {
    const float cs = etq_s[L.f0 + e].x;             // cos(TQ theta_f)
    L.twoc[e] = make_float2(2.f * cs, 2.f * cs);
    L.mtwoc[e] = make_float2(-2.f * cs, -2.f * cs);
  }
}

// Scores of the warp's kPPW pages of a chunk (kPPW * 8 tokens).  Lane (tq, P)
// owns pair-group P and, in page pi, the tokens tq + TQ i (i < TPL): n = pi TPL + i
// counts its NP = kPPW TPL tokens.  It accumulates each token's partial dot
// product over its pair-group; one transposed reduction over the NP lanes of a
// token phase then leaves lane (tq, P) with the full score of its own token,
// n = P: page P / TPL, token tq + TQ (P % TPL).
// The recurrence state (Wc, Wn) holds X_n = s_n W_n and X_{n+1}, s_n = +1, +1,
// -1, -1, ... (period 4): X_{n+2} = k X_{n+1} + X_n with k = +2 cos(s theta)
// for odd n and -2 cos(s theta) for even n -- no negated operand -- and token n
// scores s_n times the dot product with X_n.  On return the state has moved on by
// NP tokens.
template <int D, int C>
__device__ inline float run_scores(const Lane<D, C>& L, const unsigned char* Ks, const unsigned char* pages,
                                   float2 (&Wc)[Dec<D, C>::CL], float2 (&Wn)[Dec<D, C>::CL]) {
  using X = Dec<D, C>;
  constexpr int TQ = X::TQ, TPL = X::TPL, NP = X::NP, NPV = X::NPV, CL = X::CL;
  static_assert(kPPW * TPL == NPV, "one token per lane after the reduction");
  float acc[NPV];
#pragma unroll
  for (int pi = 0; pi < kPPW; ++pi) {
    const unsigned char* pg = pages + pi * X::PAGE;
    const uint2 wlo = *reinterpret_cast<const uint2*>(pg + L.P * kPage);
    const uint2 whi = *reinterpret_cast<const uint2*>(pg + (L.P + NP) * kPage);
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const int n = pi * TPL + i;                    // compile-time
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
      uint32_t lo[CL / 2], hi[CL / 2];
      load_row<CL>(Ks, row_addr<D>(xl, L.gb_lo, sel), lo);
      load_row<CL>(Ks, row_addr<D>(xh, L.gb_hi, sel), hi);
      float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int w = 0; w < CL / 2; ++w) {
        a2 = __ffma2_rn(Wc[2 * w], make_float2(bf16_lo(lo[w]), bf16_lo(hi[w])), a2);
        a2 = __ffma2_rn(Wc[2 * w + 1], make_float2(bf16_hi(lo[w]), bf16_hi(hi[w])), a2);
      }
      acc[n] = (n & 2) ? -a2.x - a2.y : a2.x + a2.y;
#pragma unroll
      for (int e = 0; e < CL; ++e) {
        const float2 nx = __ffma2_rn((n & 1) ? L.twoc[e] : L.mtwoc[e], Wn[e], Wc[e]);
        Wc[e] = Wn[e];
        Wn[e] = nx;
      }
    }
  }
  // transposed reduction over the NPV lanes of a token phase: at each level a lane
  // keeps the half of its values selected by bit o of vp and adds its partner's
#pragma unroll
  for (int o = NPV / 2; o > 0; o >>= 1) {
    const bool up = (L.vp & o) != 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float send = up ? acc[k] : acc[k + o];
      const float keep = up ? acc[k + o] : acc[k];
      acc[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return acc[0];
}

// A request's counters and the coded token range [n0, n1) of split j of ns (one split per
// ceil(Lc / ns) tokens, rounded up to 32).  `bad`: counters outside the cache's capacity.
struct SplitRange {
  bool bad;
  int S_eff, recent, n0, n1;
};
__device__ inline SplitRange split_range(const Geo& g, int ctx, int Lc, int j, int ns) {
  SplitRange r;
  r.S_eff = min(g.S, max(ctx, 0));
  r.recent = ctx - r.S_eff - Lc;
  r.bad = ctx < 1 || ctx > g.max_ctx || Lc < 0 || Lc > g.P * kPage || (Lc > 0 && ctx < g.S + Lc) || r.recent < 0 ||
          r.recent > g.R;
  int chunk = (Lc + ns - 1) / ns;
  chunk = (chunk + 31) & ~31;
  r.n0 = r.bad ? 0 : min(Lc, j * chunk);
  r.n1 = r.bad ? 0 : min(Lc, r.n0 + chunk);
  return r;
}

__device__ inline void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(src), "r"(bytes) : "memory");
}

// Programmatic dependent launch: wait until the preceding kernel of the stream
// has completed and its writes are visible; let the next kernel launch early.
// Without a programmatic predecessor or successor both are no-ops.
__device__ inline void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Barrier of the compute warps only (the producer warp never joins it).
__device__ inline void compute_sync() {
  asm volatile("bar.sync %0, %1;" :: "r"(kBarCompute), "r"(kCT) : "memory");
}
// The same barrier, returning the OR of `v` over the compute threads.
__device__ inline bool compute_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r) : "r"((uint32_t)v), "r"(kBarCompute), "r"(kCT) : "memory");
  return r != 0;
}

__device__ inline uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ inline void red_add_shared(uint32_t addr, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

// Adds the weights of the lane's value tokens of one page to the histogram:
// H[code][g] += w.  `pg` points at the lane's first code byte, `pw` at its
// first weight; `hl` is the shared address of H[0][g].
template <int D, int C>
__device__ inline void hist_page(const unsigned char* pg, const uint32_t* pw, uint32_t hl) {
  using X = Dec<D, C>;
  constexpr int VPL = X::VPL, SH = X::SH;
  uint32_t cw[2], w[8];
  if constexpr (VPL == 8) {
    const uint2 c = *reinterpret_cast<const uint2*>(pg);
    cw[0] = c.x; cw[1] = c.y;
    const uint4 a = *reinterpret_cast<const uint4*>(pw);
    const uint4 b = *reinterpret_cast<const uint4*>(pw + 4);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else if constexpr (VPL == 4) {
    cw[0] = *reinterpret_cast<const uint32_t*>(pg);
    const uint4 a = *reinterpret_cast<const uint4*>(pw);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
  } else {
    cw[0] = *reinterpret_cast<const uint16_t*>(pg);
    const uint2 a = *reinterpret_cast<const uint2*>(pw);
    w[0] = a.x; w[1] = a.y;
  }
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const uint32_t code = __byte_perm(cw[k >> 2], 0u, 0x4440u | (uint32_t)(k & 3));
    red_add_shared(hl + (code << SH), w[k]);
  }
}

// Non-blocking test of an mbarrier phase.
__device__ inline bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

constexpr int kBf16Batch = 60;               // bf16 tokens staged at once in the value-slice area

// This CTA's share of the bf16 tokens (list entries j, j + ns, ... of [sink tokens,
// recent tokens]), computed by one warp.  Per batch of up to 60 tokens the key and
// value rows and the coarse RoPE rows of their positions, plus (once) the fine RoPE
// rows, are bulk-copied into `area` (the value-slice area, free until then); the
// warp scores each token against the query rotated to its position, keeps an online
// softmax across batches and writes the partial (o, m, l) to `part`.  Returns true if
// a wait timed out (the outcome is uniform over the warp).  misc[4] counts the
// batches whose copies were issued.  `service()` is called between the steps (and
// while the copies are awaited) so that the warp keeps feeding the code-page ring.
template <int D, int C, class Service>
__device__ bool bf16_share(Service& service, const Geo& g, int layer, int step, int b, int h, int j, int ns, int S_eff, int Lc,
                           int nbj, const __nv_bfloat16* __restrict__ sink, const __nv_bfloat16* __restrict__ ring,
                           const float* __restrict__ rope, const float2* zq, unsigned char* area, uint32_t bar,
                           float* part, int* misc, long wait_iters) {
  constexpr int F = D / 2, FPL = F / 32, CPL = D / 32, BB = kBf16Batch;
  static_assert(8 * F * 8 + BB * (F * 8 + 4 * D) <= kEntries * D * 2, "bf16 batch fits the value-slice area");
  const int lane = threadIdx.x & 31;
  float2* fine_s = reinterpret_cast<float2*>(area);                        // [8][F]
  float2* coarse_s = fine_s + 8 * F;                                       // [BB][F]
  __nv_bfloat16* kb = reinterpret_cast<__nv_bfloat16*>(coarse_s + BB * F);  // [BB][D]
  __nv_bfloat16* vb = kb + BB * D;                                         // [BB][D]
  auto pos_of = [&](int k) { const int i = j + k * ns; return i < S_eff ? i : g.S + Lc + (i - S_eff); };
  auto row_of = [&](int k, int kv) -> const __nv_bfloat16* {
    const int i = j + k * ns;
    if (i < S_eff) return sink + sink_off(g, layer, kv, step, b, h, i);
    return ring + ring_off(g, layer, kv, step, b, h, (pos_of(k) - g.S) % g.R);
  };
  bool to = false;
  float m = -INFINITY, l = 0.f, o[CPL];
#pragma unroll
  for (int u = 0; u < CPL; ++u) o[u] = 0.f;
  int batch = 0;
  for (int k0 = 0; k0 < nbj && !to; k0 += BB, ++batch) {
    const int nbb = min(BB, nbj - k0);
    if (batch > 0) fence_proxy_async_shared();          // this warp's reads of the area precede the new copies
    if (lane == 0) {
      mbar_expect_tx(bar, (batch == 0 ? 8 * F * 8 : 0) + nbb * (F * 8 + 4 * D));
      misc[4] = batch + 1;
    }
    __syncwarp();
    if (batch == 0 && lane == 0)
      bulk_g2s(smem_addr(fine_s), rope + (size_t)g.RC * F * 2, 8 * F * 8, bar);
    for (int k = lane; k < nbb; k += 32) {
      bulk_g2s(smem_addr(coarse_s + k * F), rope + (size_t)(pos_of(k0 + k) >> 3) * F * 2, F * 8, bar);
      bulk_g2s(smem_addr(kb + k * D), row_of(k0 + k, 0), D * 2, bar);
      bulk_g2s(smem_addr(vb + k * D), row_of(k0 + k, 1), D * 2, bar);
    }
    {
      bool done = false;
      for (long it = 0; it < wait_iters && !done; ++it) {
        done = __all_sync(0xffffffffu, mbar_test(bar, batch & 1));
        if (!done) service();
      }
      to = !done;
    }
    if (to) break;
    service();
    // scores: four tokens at a time, lanes over frequencies; lane (k % 32) keeps token k's
    float sc0 = -INFINITY, sc1 = -INFINITY;
    for (int k4 = 0; k4 < nbb; k4 += 4) {
      float acc[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int k = min(k4 + t, nbb - 1);
        const int p7 = pos_of(k0 + k) & 7;
        acc[t] = 0.f;
#pragma unroll
        for (int u = 0; u < FPL; ++u) {
          const int f = lane + 32 * u;
          const float2 w = cmul(zq[f], cconj(cmul(coarse_s[k * F + f], fine_s[p7 * F + f])));
          acc[t] = fmaf(w.x, __bfloat162float(kb[k * D + f]), acc[t]);
          acc[t] = fmaf(w.y, __bfloat162float(kb[k * D + f + F]), acc[t]);
        }
      }
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1)
#pragma unroll
        for (int t = 0; t < 4; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o2);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int k = k4 + t;
        if (k < nbb && (k & 31) == lane) {
          if (k < 32) sc0 = acc[t];
          else sc1 = acc[t];
        }
        service();
      }
    }
    // online softmax across batches
    const float m_new = fmaxf(m, warp_max(fmaxf(sc0, sc1)));
    const float a_old = l > 0.f ? exp2f(m - m_new) : 0.f;
    const float p0 = lane < nbb ? exp2f(sc0 - m_new) : 0.f;
    const float p1 = lane + 32 < nbb ? exp2f(sc1 - m_new) : 0.f;
    l = l * a_old + warp_sum(p0 + p1);
#pragma unroll
    for (int u = 0; u < CPL; ++u) o[u] *= a_old;
    for (int k = 0; k < nbb; ++k) {
      const float pk = __shfl_sync(0xffffffffu, k < 32 ? p0 : p1, k & 31);
#pragma unroll
      for (int u = 0; u < CPL; ++u) o[u] = fmaf(pk, __bfloat162float(vb[k * D + lane + 32 * u]), o[u]);
      if ((k & 3) == 3) service();
    }
    m = m_new;
    service();
  }
  fence_proxy_async_shared();                           // the value slice is copied into the area next
  __syncwarp();
#pragma unroll
  for (int u = 0; u < CPL; ++u) part[lane + 32 * u] = to ? 0.f : o[u];
  if (lane == 0) {
    part[D] = to || l == 0.f ? -INFINITY : m;
    part[D + 1] = to ? 0.f : l;
  }
  return to;
}

// A compute warp's part of an item's bf16 share (list entries j, j + ns, ... of [sink tokens,
// recent tokens]) when CTAs walk runs of items: tokens w, w + nw, w + 2 nw, ... of the share,
// read straight from global memory (prefetched into L2 by the producer when the item began).  Lane l owns the frequencies f = l FPL + u (u < FPL) and the value channels l CPL + u
// (u < CPL).  Per group of kShareGroup tokens every lane loads its key pairs (k_f, k_{f+d/2}),
// the coarse and fine RoPE factors of the token's position and its value channels; the warp
// scores the tokens against the query rotated to its own position (zq), keeps an online softmax
// and writes its partial (o, m, l) to `part`.
constexpr int kShareGroup = 2;
template <int D>
__device__ void share_warp(const Geo& g, int layer, int step, int b, int h, int j, int ns, int S_eff, int Lc,
                           int nbj, const __nv_bfloat16* __restrict__ sink, const __nv_bfloat16* __restrict__ ring,
                           const float* __restrict__ rope, const float2* zq, int w, int nw, float* part) {
  constexpr int F = D / 2, FPL = F / 32, CPL = D / 32, TB = kShareGroup;
  static_assert(FPL == 1 || FPL == 2, "frequencies per lane");
  static_assert(CPL == 2 || CPL == 4, "value channels per lane");
  const int lane = threadIdx.x & 31;
  auto pos_of = [&](int k) { const int i = j + k * ns; return i < S_eff ? i : g.S + Lc + (i - S_eff); };
  auto row_of = [&](int k, int kv) -> const __nv_bfloat16* {
    const int i = j + k * ns;
    if (i < S_eff) return sink + sink_off(g, layer, kv, step, b, h, i);
    return ring + ring_off(g, layer, kv, step, b, h, (pos_of(k) - g.S) % g.R);
  };
  using KW = std::conditional_t<FPL == 2, uint32_t, unsigned short>;
  using VW = std::conditional_t<CPL == 4, uint2, uint32_t>;
  using RW = std::conditional_t<FPL == 2, float4, float2>;
  float2 zr[FPL];
#pragma unroll
  for (int u = 0; u < FPL; ++u) zr[u] = zq[lane * FPL + u];
  float m = -INFINITY, l = 0.f, o[CPL];
#pragma unroll
  for (int u = 0; u < CPL; ++u) o[u] = 0.f;
  for (int k0 = w; k0 < nbj; k0 += TB * nw) {
    RW ec[TB], ef[TB];
    KW klo[TB], khi[TB];
    VW vv[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      int k = k0 + t * nw;
      if (k >= nbj) k = k0;                           // past the share's end: a repeat, masked below
      const int p = pos_of(k);
      const __nv_bfloat16* kr = row_of(k, 0);
      ec[t] = __ldg(reinterpret_cast<const RW*>(rope + ((size_t)(p >> 3) * F + lane * FPL) * 2));
      ef[t] = __ldg(reinterpret_cast<const RW*>(rope + ((size_t)(g.RC + (p & 7)) * F + lane * FPL) * 2));
      klo[t] = __ldg(reinterpret_cast<const KW*>(kr + lane * FPL));
      khi[t] = __ldg(reinterpret_cast<const KW*>(kr + F + lane * FPL));
      vv[t] = __ldg(reinterpret_cast<const VW*>(row_of(k, 1) + lane * CPL));
    }
    float sc[TB];
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      float2 c[FPL], f2[FPL];
      float kl[FPL], kh[FPL];
      if constexpr (FPL == 2) {
        c[0] = make_float2(ec[t].x, ec[t].y); c[1] = make_float2(ec[t].z, ec[t].w);
        f2[0] = make_float2(ef[t].x, ef[t].y); f2[1] = make_float2(ef[t].z, ef[t].w);
        kl[0] = bf16_lo(klo[t]); kl[1] = bf16_hi(klo[t]);
        kh[0] = bf16_lo(khi[t]); kh[1] = bf16_hi(khi[t]);
      } else {
        c[0] = ec[t];
        f2[0] = ef[t];
        kl[0] = __uint_as_float((uint32_t)klo[t] << 16);
        kh[0] = __uint_as_float((uint32_t)khi[t] << 16);
      }
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < FPL; ++u) {
        const float2 wq = cmul(zr[u], cconj(cmul(c[u], f2[u])));
        acc = fmaf(wq.x, kl[u], acc);
        acc = fmaf(wq.y, kh[u], acc);
      }
      sc[t] = acc;
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1)
#pragma unroll
      for (int t = 0; t < TB; ++t) sc[t] += __shfl_xor_sync(0xffffffffu, sc[t], o2);
    float mg = -INFINITY;
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      if (k0 + t * nw >= nbj) sc[t] = -INFINITY;
      mg = fmaxf(mg, sc[t]);
    }
    const float m_new = fmaxf(m, mg);
    const float a_old = l > 0.f ? exp2f(m - m_new) : 0.f;
    float pt[TB], ps = 0.f;
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      pt[t] = k0 + t * nw < nbj ? exp2f(sc[t] - m_new) : 0.f;
      ps += pt[t];
    }
    l = l * a_old + ps;
#pragma unroll
    for (int u = 0; u < CPL; ++u) o[u] *= a_old;
#pragma unroll
    for (int t = 0; t < TB; ++t) {
      float v[CPL];
      if constexpr (CPL == 4) {
        v[0] = bf16_lo(vv[t].x); v[1] = bf16_hi(vv[t].x); v[2] = bf16_lo(vv[t].y); v[3] = bf16_hi(vv[t].y);
      } else {
        v[0] = bf16_lo(vv[t]); v[1] = bf16_hi(vv[t]);
      }
#pragma unroll
      for (int u = 0; u < CPL; ++u) o[u] = fmaf(pt[t], v[u], o[u]);
    }
    m = m_new;
  }
#pragma unroll
  for (int u = 0; u < CPL; ++u) part[lane * CPL + u] = o[u];
  if (lane == 0) {
    part[D] = l == 0.f ? -INFINITY : m;
    part[D + 1] = l;
  }
}

// L2 prefetch, by the lanes of one warp, of the rows an item's bf16 share reads (key, value and
// coarse RoPE rows of its first 64 tokens), so that the compute warps' loads find them in L2.
// The counters may be hints: split_range's checks keep every address inside the sink, ring and
// RoPE buffers.
template <int D>
__device__ inline void prefetch_share(const Geo& g, int layer, int step, int b, int h, int j, int ns, int ctx, int Lc,
                                      const __nv_bfloat16* sink, const __nv_bfloat16* ring, const float* rope) {
  constexpr int F = D / 2;
  const SplitRange r = split_range(g, ctx, Lc, j, ns);
  const int nb = r.bad ? 0 : r.S_eff + r.recent;
  const int nbj = nb > j ? min(64, (nb - j + ns - 1) / ns) : 0;
  for (int k = threadIdx.x & 31; k < nbj; k += 32) {
    const int i = j + k * ns;
    const int p = i < r.S_eff ? i : g.S + Lc + (i - r.S_eff);
    for (int kv = 0; kv < 2; ++kv)
      prefetch_l2_bulk(i < r.S_eff ? sink + sink_off(g, layer, kv, step, b, h, i)
                                   : ring + ring_off(g, layer, kv, step, b, h, (p - g.S) % g.R),
                       D * 2);
    prefetch_l2_bulk(rope + (size_t)(p >> 3) * F * 2, F * 8);
  }
}

// decode_runs_kernel: the last item of a (request, query head) to finish merges its 2 ns partials
// (coded split j at slot 2j, bf16 share of split j at 2j + 1) by logsumexp, with the compute
// threads: out, lse, the per-split LSEs, and the merge counter returned to zero.  `scr` is shared
// scratch (the score array).
template <int D>
__device__ void merge_partials(const float* ws, size_t slot0, int ns, float* out, float* lse, float* sl,
                               int32_t* counter, float* scr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __threadfence();
  const int np = 2 * ns;
  const float* base = ws + slot0 * (D + 2);
  constexpr int RB = kCT / D;                 // partial phases of the output sum
  constexpr int MPF = 8;                      // output elements prefetched per thread
  const int e = tid % D, r = tid / D;
  const bool act = r < RB;
  // every load is issued before the first use: o[e] of partials r, r + RB, ...
  float opre[MPF];
#pragma unroll
  for (int u = 0; u < MPF; ++u) {
    const int i = r + RB * u;
    opre[u] = act && i < np ? __ldcg(base + (size_t)i * (D + 2) + e) : 0.f;
  }
  float* pl2 = scr;             // [np] partial LSEs (log2)
  float* pw = scr + 512;        // [np] partial maxima, then weights
  for (int i = tid; i < np; i += kCT) {
    const float pm = __ldcg(base + (size_t)i * (D + 2) + D), pl = __ldcg(base + (size_t)i * (D + 2) + D + 1);
    pl2[i] = pl > 0.f ? pm + log2f(pl) : -INFINITY;
    pw[i] = pm;
  }
  compute_sync();
  // warp 0: the LSE over the partials and every partial's weight 2^(m_i - L)
  float Ltot = -INFINITY;
  if (warp == 0) {
    float M = -INFINITY;
    for (int i = lane; i < np; i += 32) M = fmaxf(M, pl2[i]);
    M = warp_max(M);
    float den = 0.f;
    if (M != -INFINITY)
      for (int i = lane; i < np; i += 32)
        if (pl2[i] != -INFINITY) den += exp2f(pl2[i] - M);
    den = warp_sum(den);
    Ltot = M == -INFINITY ? -INFINITY : M + log2f(den);
    for (int i = lane; i < np; i += 32) pw[i] = pl2[i] == -INFINITY ? 0.f : exp2f(pw[i] - Ltot);
  }
  compute_sync();
  float* rb = scr + 1024;       // [RB][D]
  if (act) {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < MPF; ++u) {
      const int i = r + RB * u;
      if (i < np) acc = fmaf(pw[i], opre[u], acc);
    }
    for (int i = r + RB * MPF; i < np; i += RB) acc = fmaf(pw[i], __ldcg(base + (size_t)i * (D + 2) + e), acc);
    rb[r * D + e] = acc;
  }
  compute_sync();
  if (tid < D) {
    float t = 0.f;
#pragma unroll
    for (int r2 = 0; r2 < RB; ++r2) t += rb[r2 * D + tid];
    out[tid] = t;
  }
  constexpr float kLn2 = 0.6931471805599453f;
  if (warp == 0) {
    if (lane == 0) {
      *lse = Ltot * kLn2;
      *counter = 0;
    }
    if (sl) {
      for (int i = lane; i < ns; i += 32) sl[i] = pl2[2 * i] * kLn2;
      // the bf16 partial is the logsumexp of the items' shares
      float Bm = -INFINITY;
      for (int i = lane; i < ns; i += 32) Bm = fmaxf(Bm, pl2[2 * i + 1]);
      Bm = warp_max(Bm);
      float Bs = 0.f;
      if (Bm != -INFINITY)
        for (int i = lane; i < ns; i += 32)
          if (pl2[2 * i + 1] != -INFINITY) Bs += exp2f(pl2[2 * i + 1] - Bm);
      Bs = warp_sum(Bs);
      if (lane == 0) sl[ns] = Bm == -INFINITY ? -INFINITY : (Bm + log2f(Bs)) * kLn2;
    }
  }
  compute_sync();               // the scratch is the next item's score array
}

// Work items of one launch: (request b, query head hq, split j), ordered by KV head, then
// request, then split, then the query heads of the KV head:
//   it = ((h * batch + b) * ns + j) * gq + r,   hq = h * gq + r,   gq = Hq / H.
// A CTA takes a contiguous run of items, so consecutive items share the KV head (its step
// slices stay in shared memory) and, with several query heads per KV head, the code pages
// (read again from L2).
struct Item {
  int b, hq, h, j;
};
__device__ inline Item item_at(int it, int batch, int ns, int gq) {
  Item x;
  int t = it / gq;
  const int r = it - t * gq;
  x.j = t % ns;
  t /= ns;
  x.b = t % batch;
  x.h = t / batch;
  x.hq = x.h * gq + r;
  return x;
}

constexpr int kItemCost = 1200;  // per-item overhead of the balanced partition, in coded tokens

// Launches with fewer CTAs than items (one CTA per SM): CTA c of G takes the items whose cost
// midpoint P + cost / 2 (P: the cost of the items before it, cost: its coded tokens plus
// kItemCost, in item order) has floor((P + cost / 2) G / total) = c, a contiguous run balanced
// to within an item.  One warp computes it from the counters, staged in
// `scr` (16 bytes per request, plus 8); every CTA computes the same partition.
__device__ inline void partition_items(const Geo& g, const int32_t* ctx_len, const int32_t* coded_len, int batch,
                                       int ns, int c, int G, unsigned char* scr, int& it0, int& it1) {
  const int lane = threadIdx.x & 31, gq = g.Hq / g.H;
  long long* pre = reinterpret_cast<long long*>(scr);     // [batch + 1] exclusive prefix of request costs
  int* cx = reinterpret_cast<int*>(pre + batch + 1);      // [batch] context lengths
  int* lc = cx + batch;                                   // [batch] coded lengths
  for (int b = lane; b < batch; b += 32) {
    const int x = ctx_len[b], l = coded_len[b];
    cx[b] = x;
    lc[b] = l;
    const SplitRange r = split_range(g, x, l, 0, ns);
    pre[b] = (long long)gq * ((r.bad ? 0 : l) + (long long)ns * kItemCost);
  }
  __syncwarp();
  if (lane == 0) {
    long long acc = 0;
    for (int b = 0; b < batch; ++b) {
      const long long v = pre[b];
      pre[b] = acc;
      acc += v;
    }
    pre[batch] = acc;
  }
  __syncwarp();
  const long long W = pre[batch], total = W * g.H;      // > 0: every item costs at least kItemCost
  const int N = g.H * batch * ns * gq;
  auto owner = [&](int it) {
    const Item x = item_at(it, batch, ns, gq);
    const SplitRange r = split_range(g, cx[x.b], lc[x.b], x.j, ns);
    const long long cost = (long long)(r.n1 - r.n0) + kItemCost;
    const long long P = x.h * W + pre[x.b] + gq * ((long long)r.n0 + (long long)x.j * kItemCost) +
                        (long long)(x.hq - x.h * gq) * cost;
    return (int)min((long long)(G - 1), (2 * P + cost) * G / (2 * total));   // by the item's midpoint
  };
  // the first item whose owner is >= cc (N if none), by a 32-way search: [lo, hi] holds it
  auto first_owned = [&](int cc) {
    int lo = 0, hi = N;
    while (lo < hi) {
      const int stride = (hi - lo + 31) / 32;
      const int probe = lo + lane * stride;
      const uint32_t m = __ballot_sync(0xffffffffu, probe >= hi || owner(probe) >= cc);
      if (m == 0u) {
        lo += 31 * stride + 1;
      } else {
        const int f = __ffs(m) - 1;
        if (f == 0) {
          hi = lo;
        } else {
          hi = min(hi, lo + f * stride);
          lo += (f - 1) * stride + 1;
        }
      }
    }
    return lo;
  };
  it0 = first_owned(c);
  it1 = first_owned(c + 1);
}

// Per-item geometry: counters, coded range and stream shape (the same on both roles).
struct ItemGeo {
  Item x;
  SplitRange sr;
  int ctx, Lc, n_kchunks, n_stream, n_super, nbj;
  bool do_coded;
};
template <int D, int C>
__device__ inline ItemGeo item_geo(const Geo& g, int it, int batch, int ns, const int32_t* ctx_len,
                                   const int32_t* coded_len) {
  using X = Dec<D, C>;
  ItemGeo e;
  e.x = item_at(it, batch, ns, g.Hq / g.H);
  e.ctx = ctx_len[e.x.b];
  e.Lc = coded_len[e.x.b];
  e.sr = split_range(g, e.ctx, e.Lc, e.x.j, ns);
  e.do_coded = e.sr.n0 < e.sr.n1;
  e.n_kchunks = e.do_coded ? (e.sr.n1 - e.sr.n0 + kChunk - 1) / kChunk : 0;
  e.n_stream = 2 * e.n_kchunks;                 // per super-chunk: its K chunks, then its V chunks
  e.n_super = e.do_coded ? (e.sr.n1 - e.sr.n0 + X::NSC - 1) / X::NSC : 0;
  const int nb = e.sr.bad ? 0 : e.sr.S_eff + e.sr.recent;          // bf16 tokens: [sink, recent]
  e.nbj = nb > e.x.j ? (nb - e.x.j + ns - 1) / ns : 0;              // the item's share: j, j + ns, ...
  return e;
}

// DBG: the instantiation used while the test hook is active (its wait bound and fault bits
// come from the geometry); the normal ones keep the constant bound.  PM: 0 per-request code
// streams, 1 pool mode, -1 either (read from the geometry; the test-hook instantiation).
template <int D, int C, bool DBG, int PM>
__global__ void __launch_bounds__(kThr, 1) decode_kernel(
    Geo g, int layer, int step, const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ ctx_len,
    const int32_t* __restrict__ coded_len, const __nv_bfloat16* __restrict__ sink,
    const __nv_bfloat16* __restrict__ ring, const uint8_t* __restrict__ idx,
    const __nv_bfloat16* __restrict__ cbp, const float* __restrict__ rope, int ns,
    float* __restrict__ ws, float* __restrict__ out, float* __restrict__ lse, float* __restrict__ split_lse,
    int32_t* st) {
  using X = Dec<D, C>;
  const long wit = DBG ? g.wait_iters : kWaitIters;   // bound of every wait
  const bool pool = PM < 0 ? g.pool != 0 : PM != 0;
  constexpr int F = X::F, NG = X::NG, TQ = X::TQ, NPAIR = X::NPAIR, NREP = X::NREP;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* Ks = smem;
  const unsigned char* Vsm = smem + X::OFF_V;
  uint32_t* Hs = reinterpret_cast<uint32_t*>(smem + X::OFF_H);
  unsigned char* ringb = smem + X::OFF_RING;
  float2* zq = reinterpret_cast<float2*>(smem + X::OFF_ZQ);
  float2* etq_s = reinterpret_cast<float2*>(smem + X::OFF_TAB);       // [F] e^{-i TQ theta_f}
  float2* ech_s = etq_s + F;                                           // [F] e^{-i kChunk theta_f}
  float* red = reinterpret_cast<float*>(smem + X::OFF_RED);
  // misc: [0] failure, [1] merger, [2] chunks issued, [3] V slice issued, [4] bf16 batches issued
  int* misc = reinterpret_cast<int*>(smem + X::OFF_MISC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);
  float* SC = reinterpret_cast<float*>(smem + X::OFF_SC);    // scores, then weights; scratch elsewhere
  // bars[0]: K slice; bars[1]: V slice; bars[2 + s]: stage s full; bars[2 + kStages + s]: stage s empty;
  // bars[2 + 2 kStages]: the bf16 rows

  const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int h = hq / (g.Hq / g.H);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == kCW;
  const int blk = step / g.Tc, s = step % g.Tc;
  const size_t slot0 = ((size_t)b * g.Hq + hq) * g.max_splits * 2;        // partial slots [split][coded, bf16]
  float* part_coded = ws + (slot0 + 2 * j) * (D + 2);
  float* part_bf16 = ws + (slot0 + 2 * j + 1) * (D + 2);
  int32_t* counters = reinterpret_cast<int32_t*>(ws + (size_t)g.B * g.Hq * g.max_splits * 2 * (D + 2));

  if (tid == 0) {
    for (int i = 0; i < X::NBAR; ++i) mbar_init(smem_addr(&bars[i]), i >= 2 + kStages && i < 2 + 2 * kStages ? kCW : 1);
    fence_mbar_init();
    misc[0] = 0;
    misc[1] = 0;
    misc[2] = 0;
    misc[3] = 0;
    misc[4] = 0;
  }
  __syncthreads();
  // The step-t key slice depends on nothing another kernel of a decode sequence writes, so it is
  // fetched before waiting for the preceding kernel in the stream (programmatic dependent launch):
  // its latency overlaps that kernel's tail.  Everything else is read after the wait.  Before it,
  // the counters are read only as a hint (the preceding kernel may still rewrite them; read
  // through L2, not kept in L1): the split's first key pages and RoPE rows they name are prefetched
  // into L2, always inside the request's own stream and the RoPE table, so the real copies issued
  // after the wait find them there.
  if (producer && lane == 0) {
    const uint32_t bk = smem_addr(&bars[0]);
    mbar_expect_tx(bk, X::KS);
    bulk_g2s(smem_addr(Ks), cbp + cbp_slice_off(g, layer, 0, blk, h, s), X::KS, bk);
    if (!pool) {
      const SplitRange hint = split_range(g, __ldcg(ctx_len + b), __ldcg(coded_len + b), j, ns);
      if (hint.n0 < hint.n1) {
        const int t1 = min(hint.n1, hint.n0 + kStages * kChunk);
        prefetch_l2_bulk(idx + idx_stream_off(g, layer, blk, b, h, 0) + (size_t)(hint.n0 / kPage) * X::PAGE,
                         (uint32_t)((t1 - hint.n0 + kPage - 1) / kPage) * X::PAGE);
        const int r0 = (g.S + hint.n0) >> 3, r1 = (g.S + min(hint.n1, hint.n0 + kChunk) - 1) >> 3;
        prefetch_l2_bulk(rope + (size_t)r0 * F * 2, (uint32_t)(r1 - r0 + 1) * F * 8);
      }
    }
  }
  grid_dependency_wait();
  launch_dependents();

  const int ctx = ctx_len[b], Lc = coded_len[b];
  const SplitRange sr = split_range(g, ctx, Lc, j, ns);
  const bool bad = sr.bad;
  const int S_eff = sr.S_eff, recent = sr.recent, n0 = sr.n0, n1 = sr.n1;
  if (bad && j == 0 && tid == 0) set_status(st, LVQ_ECAPACITY);
  const bool do_coded = n0 < n1;
  const int n_kchunks = do_coded ? (n1 - n0 + kChunk - 1) / kChunk : 0;
  const int n_stream = 2 * n_kchunks;            // per super-chunk: its K chunks, then its V chunks
  const int n_super = do_coded ? (n1 - n0 + X::NSC - 1) / X::NSC : 0;
  constexpr int CPS = X::NSC / kChunk;           // chunks per full super-chunk
  // per-request streams: the K pages, then the V pages, of (layer, blk, b, h); pool mode: the pools
  // of (layer, blk, h), the request's pages found through the page table
  const uint8_t* kstream = idx + (pool ? idx_pool_off(g, layer, blk, h, 0) : idx_stream_off(g, layer, blk, b, h, 0));
  const uint8_t* vstream = idx + (pool ? idx_pool_off(g, layer, blk, h, 1) : idx_stream_off(g, layer, blk, b, h, 1));

  // the V slice is needed only by the first contraction: the producer copies it once its bf16 share
  // (staged in the same area) is done
  auto issue_v_slice = [&]() {
    const uint32_t bv = smem_addr(&bars[1]);
    mbar_expect_tx(bv, X::KS);
    bulk_g2s(smem_addr(Vsm), cbp + cbp_slice_off(g, layer, 1, blk, h, s), X::KS, bv);
  };
  // first coded token, pages and K/V side of chunk ci
  auto chunk_geom = [&](int ci, int& c0, int& np, bool& is_v) {
    const int sc = ci / (2 * CPS), r = ci % (2 * CPS);
    const int nk = min(CPS, n_kchunks - sc * CPS);
    is_v = r >= nk;
    c0 = n0 + (sc * CPS + (is_v ? r - nk : r)) * kChunk;
    np = (min(n1, c0 + kChunk) - c0 + kPage - 1) / kPage;
  };
  // pool mode: the page ids of the next chunk to issue are loaded one chunk ahead (lane l holds
  // the chunk's pages l and l + 32) and range-checked only when they are used, so that the page
  // table's latency overlaps the ring's wait instead of stalling the producer
  int pf_ci = -1, pf_id[2] = {0, 0};
  const int32_t* pt_row = pool ? g.pt + (size_t)b * g.pts : nullptr;
  auto fetch_ids = [&](int ci) {
    int c0, np;
    bool v;
    chunk_geom(ci, c0, np, v);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = lane + 32 * hh;
      pf_id[hh] = i < np ? __ldg(pt_row + c0 / kPage + i) : 0;
    }
    pf_ci = ci;
  };
  // issue chunk ci.  Per-request streams: lane 0 alone, one bulk copy of the chunk's pages.  Pool
  // mode: the whole producer warp; lane l looks up the chunk's pages l and l + 32 in the page
  // table, and every run of consecutive physical pages (within a half) is one bulk copy, issued by
  // the lane at its start; an out-of-range entry is reported and page 0 copied in its place (so
  // that the stage still fills).
  auto issue_chunk = [&](int ci) {
    if (DBG && (g.fault & kFaultDecodeDropChunk) && ci == 0) return;   // test hook: this copy never happens
    int c0, np;
    bool is_v;
    chunk_geom(ci, c0, np, is_v);
    const uint32_t bar = smem_addr(&bars[2 + ci % kStages]);
    const uint32_t dst = smem_addr(ringb + (ci % kStages) * X::STAGE);
    const uint8_t* src = is_v ? vstream : kstream;
    if (lane == 0) mbar_expect_tx(bar, np * X::PAGE);
    if (!pool) {
      bulk_g2s(dst, src + (size_t)(c0 / kPage) * X::PAGE, np * X::PAGE, bar);
      return;
    }
    if (pf_ci != ci) fetch_ids(ci);
    const int ids[2] = {pf_id[0], pf_id[1]};
    if (ci + 1 < n_stream) fetch_ids(ci + 1);      // in flight until the next chunk is issued
    __syncwarp();                                   // the expected bytes are set before any copy lands
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = lane + 32 * hh;                 // page of the chunk
      const int in_half = min(32, np - 32 * hh);    // pages of this half (may be <= 0)
      int id = i < np ? ids[hh] : 0;
      const bool bad = i < np && (id < 0 || id >= g.pool);
      if (bad) {
        set_status(st, LVQ_ECAPACITY);
        id = 0;
      }
      const int prev = __shfl_up_sync(0xffffffffu, id, 1);
      const bool prev_bad = __shfl_up_sync(0xffffffffu, bad, 1);
      const bool start = i < np && (lane == 0 || bad || prev_bad || id != prev + 1);
      const uint32_t starts = __ballot_sync(0xffffffffu, start);
      if (start) {
        const uint32_t later = lane < 31 ? starts >> (lane + 1) : 0u;
        const int end = later ? lane + __ffs(later) : in_half;   // lane of the next run's start
        bulk_g2s(dst + (uint32_t)i * X::PAGE, src + (size_t)id * X::PAGE, (uint32_t)(end - lane) * X::PAGE, bar);
      }
    }
  };

  // ---- prologue: the producer starts the first chunks; compute threads rotate the query (scaled so
  // that scores come out in log2 units) and clear the histogram
  const int nb = bad ? 0 : S_eff + recent;                 // bf16 tokens: [sink tokens, recent tokens]
  const int nbj = nb > j ? (nb - j + ns - 1) / ns : 0;    // this CTA's share: j, j + ns, ...
  if (producer && do_coded && (pool || lane == 0))
    for (int ci = 0; ci < min(kStages, n_stream); ++ci) issue_chunk(ci);
  // a compute lane's RoPE factors at its first coded token, fetched now so that their latency
  // overlaps the prologue
  float2 rf[X::CL];
  if (!producer && do_coded) {
    const int p_first = g.S + n0 + kPage * kPPW * warp + lane / X::NPV;
    const int f0 = lane_f0<D, C>(lane);
#pragma unroll
    for (int e = 0; e < X::CL; ++e) rf[e] = rope_at(rope, g.RC, F, p_first, f0 + e);
  }
  if (!bad && tid < F) {
    const __nv_bfloat16* qv = q + ((size_t)b * g.Hq + hq) * D;
    const float2 qraw = make_float2(__bfloat162float(qv[tid]), __bfloat162float(qv[tid + F]));
    const float2 qe = rope_at(rope, g.RC, F, ctx - 1, tid);
    const float2 e_tq = rope_at(rope, g.RC, F, X::TQ, tid);
    const float2 e_ch = rope_at(rope, g.RC, F, kChunk, tid);
    const float qscale = 1.4426950408889634f * rsqrtf((float)D);
    zq[tid] = make_float2((qraw.x * qe.x - qraw.y * qe.y) * qscale, (qraw.y * qe.x + qraw.x * qe.y) * qscale);
    etq_s[tid] = cconj(e_tq);
    ech_s[tid] = cconj(e_ch);
  }
  if (!producer)
    for (int i = tid; i < X::HB / 16; i += kCT) reinterpret_cast<uint4*>(Hs)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();

  bool timed_out = false;
  float m_run = -INFINITY, l_run = 0.f;       // the coded partial, held by compute threads tid < NPAIR
  float2 o_run = make_float2(0.f, 0.f);

  if (do_coded) {
    if (producer) {
      // ---- producer: the bf16 share, feeding the ring meanwhile (every chunk whose stage its
      // consumers have released, as lane 0 sees the stage); the V slice into the area the share
      // used; then the rest of the chunks.  The ring is fed by lane 0 (per-request streams) or by
      // the whole warp (pool mode).
      int ci_next = min(kStages, n_stream);
      auto stage_free = [&](int ci) {
        return mbar_test(smem_addr(&bars[2 + kStages + ci % kStages]), (ci / kStages - 1) & 1);
      };
      // pool mode: the ring is checked on every fourth call only (each check is a warp shuffle,
      // which waits behind the compute warps' shared-memory traffic; 561 -> 549 us per launch at
      // 32 requests)
      int svc = 0;
      auto service = [&]() {
        if (pool) {
          if ((++svc & 3) != 0) return;
          while (ci_next < n_stream && __shfl_sync(0xffffffffu, lane == 0 ? (int)stage_free(ci_next) : 0, 0))
            issue_chunk(ci_next++);
        } else if (lane == 0) {
          while (ci_next < n_stream && stage_free(ci_next)) issue_chunk(ci_next++);
        }
      };
      timed_out = bf16_share<D, C>(service, g, layer, step, b, h, j, ns, S_eff, Lc, nbj, sink, ring, rope, zq,
                                   smem + X::OFF_V, smem_addr(&bars[2 + 2 * kStages]), part_bf16, misc, wit);
      if (lane == 0 && !timed_out) {
        issue_v_slice();
        misc[3] = 1;
      }
      if (pool || lane == 0) {
        int ci = ci_next;
        for (; ci < n_stream; ++ci) {
          bool ok = mbar_wait(smem_addr(&bars[2 + kStages + ci % kStages]), (ci / kStages - 1) & 1, wit);
          if (pool) ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            timed_out = true;
            break;
          }
          issue_chunk(ci);
        }
        if (lane == 0) misc[2] = ci;
      }
    } else {
      // ---- compute warps
      Lane<D, C> L;
      lane_init<D, C>(L, lane, etq_s);
      float2 U[X::CL];                   // W of the lane's first token of the current chunk
#pragma unroll
      for (int e = 0; e < X::CL; ++e) U[e] = cmul(zq[L.f0 + e], cconj(rf[e]));
      const int pi_own = L.vp / X::TPL, t_own = L.tq + TQ * (L.vp % X::TPL);   // the lane's token of a run
      const int gv = lane % NG, tp = lane / NG;
      const uint32_t hl = smem_addr(Hs) + (uint32_t)gv * 4;
      uint32_t* PW = reinterpret_cast<uint32_t*>(SC);
      // waits are bounded; their outcome is made uniform over the warp, then over the compute warps
      timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[0]), 0, wit));
      int ci = 0;
      for (int sc = 0; sc < n_super; ++sc) {
        const int s0 = n0 + sc * X::NSC, s1 = min(n1, s0 + X::NSC);
        const int nk = (s1 - s0 + kChunk - 1) / kChunk;
        // ---- phase A: scores of the super-chunk
        float mx = -INFINITY;
        for (int kc = 0; kc < nk; ++kc, ++ci) {
          if (!timed_out)
            timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[2 + ci % kStages]), (ci / kStages) & 1,
                                                           wit));
          if (!timed_out) {
            const int c0 = s0 + kc * kChunk;
            const unsigned char* stage = ringb + (ci % kStages) * X::STAGE;
            float2 Wc[X::CL], Wn[X::CL];
#pragma unroll
            for (int e = 0; e < X::CL; ++e) {
              Wc[e] = U[e];
              Wn[e] = cmul(U[e], etq_s[L.f0 + e]);        // s_1 = +1
            }
            // pages past the split's end hold stale codes: their tokens are masked
            const float sc_ = run_scores<D, C>(L, Ks, stage + warp * kPPW * X::PAGE, Wc, Wn);
            const int tok = c0 + kPage * (warp * kPPW + pi_own) + t_own;
            const float sv = tok < s1 ? sc_ : -INFINITY;
            mx = fmaxf(mx, sv);
            SC[tok - s0] = sv;
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars[2 + kStages + ci % kStages]));
          }
#pragma unroll
          for (int e = 0; e < X::CL; ++e) U[e] = cmul(U[e], ech_s[L.f0 + e]);
        }
        // ---- weights: exact maximum, then integers round(2^(s - M) * 2^k) with 2^k * sum < 2^30
        mx = warp_max(mx);
        if (lane == 0) red[warp] = mx;
        timed_out = compute_sync_or(timed_out);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kCW; ++w) M = fmaxf(M, red[w]);
        const int len = s1 - s0, len8 = (len + kPage - 1) & ~(kPage - 1);
        float ls = 0.f;
        if (!timed_out)
#pragma unroll 4
          for (int t = tid; t < len; t += kCT) {
            const float p = exp2f(SC[t] - M);
            SC[t] = p;
            ls += p;
          }
        ls = warp_sum(ls);
        if (lane == 0) red[16 + warp] = ls;
        compute_sync();
        float Ls = 0.f;
#pragma unroll
        for (int w = 0; w < kCW; ++w) Ls += red[16 + w];
        // Ls = m 2^E with m in [0.5, 1); Ls >= 1 (the maximum's weight is 1), so 17 <= 30 - E <= 29
        const int E = ((__float_as_int(Ls) >> 23) & 0xff) - 126;
        const int kfx = min(30, max(0, 30 - E));
        const float scale = __int_as_float((127 + kfx) << 23);
        uint32_t lf = 0;
        if (!timed_out)
#pragma unroll 4
          for (int t = tid; t < len8; t += kCT) {
            const uint32_t v = t < len ? __float2uint_rn(SC[t] * scale) : 0u;
            PW[t] = v;
            lf += v;
          }
        lf = warp_sum_u32(lf);
        if (lane == 0) reinterpret_cast<uint32_t*>(red)[32 + warp] = lf;
        compute_sync();
        uint32_t Lf = 0;
#pragma unroll
        for (int w = 0; w < kCW; ++w) Lf += reinterpret_cast<uint32_t*>(red)[32 + w];
        // ---- phase B: histogram of the weights over (code, group)
        for (int kc = 0; kc < nk; ++kc, ++ci) {
          if (!timed_out)
            timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[2 + ci % kStages]), (ci / kStages) & 1,
                                                           wit));
          if (timed_out) continue;
          const int c0 = s0 + kc * kChunk;
          const unsigned char* stage = ringb + (ci % kStages) * X::STAGE;
#pragma unroll 2
          for (int pi = 0; pi < kPPW; ++pi) {
            const int pl = warp * kPPW + pi;
            const int tb = c0 + kPage * pl;
            if (tb >= s1) break;
            hist_page<D, C>(stage + pl * X::PAGE + gv * kPage + tp * X::VPL, PW + (tb - s0) + tp * X::VPL, hl);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_addr(&bars[2 + kStages + ci % kStages]));
        }
        if (!timed_out && sc == 0)
          timed_out = __any_sync(0xffffffffu, !mbar_wait(smem_addr(&bars[1]), 0, wit));
        timed_out = compute_sync_or(timed_out);
        // ---- contraction: o[ch] = sum_a H[a][ch / c] * V[a][ch], two channels per thread
        const int cp = tid % NPAIR, rep = tid / NPAIR;
        float2 acc = make_float2(0.f, 0.f);
        if (!timed_out && rep < NREP) {
          const uint32_t* vcol = reinterpret_cast<const uint32_t*>(Vsm) + cp;
          const uint32_t* hcol = Hs + (2 * cp) / C;
#pragma unroll 4
          for (int a = rep; a < kEntries; a += NREP) {
            const uint32_t v = vcol[a * NPAIR];
            const float hv = (float)hcol[a * NG];
            acc.x = fmaf(hv, bf16_lo(v), acc.x);
            acc.y = fmaf(hv, bf16_hi(v), acc.y);
          }
        }
        float2* rb = reinterpret_cast<float2*>(SC);      // [NREP][NPAIR]: the weights are no longer read
        if (rep < NREP) rb[rep * NPAIR + cp] = acc;
        compute_sync();
        if (tid < NPAIR && !timed_out && Lf > 0u) {
          float2 o = make_float2(0.f, 0.f);
#pragma unroll
          for (int r = 0; r < NREP; ++r) { o.x += rb[r * NPAIR + tid].x; o.y += rb[r * NPAIR + tid].y; }
          const float sc_scale = __int_as_float((127 - kfx) << 23);
          const float l_sc = (float)Lf * sc_scale;
          const float m_new = fmaxf(m_run, M);
          const float a_old = l_run > 0.f ? exp2f(m_run - m_new) : 0.f;
          const float a_new = exp2f(M - m_new) * sc_scale;
          o_run = make_float2(o_run.x * a_old + o.x * a_new, o_run.y * a_old + o.y * a_new);
          l_run = l_run * a_old + l_sc * exp2f(M - m_new);
          m_run = m_new;
        }
        if (sc + 1 < n_super)
          for (int i = tid; i < X::HB / 16; i += kCT) reinterpret_cast<uint4*>(Hs)[i] = make_uint4(0u, 0u, 0u, 0u);
        compute_sync();
      }
    }
  }
  auto no_service = []() {};
  if (!do_coded && producer)
    timed_out = bf16_share<D, C>(no_service, g, layer, step, b, h, j, ns, S_eff, Lc, nbj, sink, ring, rope, zq,
                                 smem + X::OFF_V, smem_addr(&bars[2 + 2 * kStages]), part_bf16, misc, wit);
  // the key slice copy was issued by every CTA: let it land before the CTA can exit
  if (tid == 0 && !do_coded && !mbar_wait(smem_addr(&bars[0]), 0, wit)) timed_out = true;
  if (__syncthreads_or(timed_out)) {
    if (tid == 0) {
      set_status(st, LVQ_ETIMEOUT);
      mbar_wait(smem_addr(&bars[0]), 0, wit);
      misc[0] = 1;
      if (do_coded) {   // let every issued copy land before the CTA can exit
        const int issued = max(misc[2], min(kStages, n_stream));
        if (misc[3]) mbar_wait(smem_addr(&bars[1]), 0, wit);
        for (int ci = max(0, issued - kStages); ci < issued; ++ci)
          mbar_wait(smem_addr(&bars[2 + ci % kStages]), (ci / kStages) & 1, wit);
      }
      if (misc[4] > 0) mbar_wait(smem_addr(&bars[2 + 2 * kStages]), (misc[4] - 1) & 1, wit);
    }
    __syncthreads();
  }
  const bool failed = misc[0] != 0;
  if (tid < NPAIR) {
    part_coded[2 * tid] = failed ? 0.f : o_run.x;
    part_coded[2 * tid + 1] = failed ? 0.f : o_run.y;
  }
  if (tid == 0) {
    part_coded[D] = failed || l_run == 0.f ? -INFINITY : m_run;
    part_coded[D + 1] = failed ? 0.f : l_run;
  }

  // ---- the last CTA of this (request, head) merges the 2 * ns partials
  __syncthreads();
  if (tid == 0) {
    __threadfence();            // this CTA's partials (ordered before by the barrier) become visible
    misc[1] = atomicAdd(&counters[(size_t)b * g.Hq + hq], 1) == ns - 1;
  }
  __syncthreads();
  if (!misc[1]) return;
  __threadfence();
  const int np = 2 * ns;
  const float* base = ws + slot0 * (D + 2);
  constexpr int RB = kThr / D;                // partial phases of the output sum
  constexpr int MPF = 8;                      // output elements prefetched per thread
  const int e = tid % D, r = tid / D;
  // every load is issued before the first use: (m, l) of partial tid, and o[e] of partials r, r + RB, ...
  float pm = -INFINITY, pl = 0.f;
  if (tid < np) {
    pm = __ldcg(base + (size_t)tid * (D + 2) + D);
    pl = __ldcg(base + (size_t)tid * (D + 2) + D + 1);
  }
  float opre[MPF];
#pragma unroll
  for (int u = 0; u < MPF; ++u) {
    const int i = r + RB * u;
    opre[u] = i < np ? __ldcg(base + (size_t)i * (D + 2) + e) : 0.f;
  }
  float* pl2 = SC;              // [np] partial LSEs (log2)
  float* pw = SC + 512;         // [np] partial weights
  if (tid < np) {
    pl2[tid] = pl > 0.f ? pm + log2f(pl) : -INFINITY;
    pw[tid] = pm;                                    // replaced by the weight below
  }
  __syncthreads();
  // warp 0: the LSE over the partials and every partial's weight 2^(m_i - L)
  float Ltot = -INFINITY;
  if (warp == 0) {
    float M = -INFINITY;
    for (int i = lane; i < np; i += 32) M = fmaxf(M, pl2[i]);
    M = warp_max(M);
    float den = 0.f;
    if (M != -INFINITY)
      for (int i = lane; i < np; i += 32)
        if (pl2[i] != -INFINITY) den += exp2f(pl2[i] - M);
    den = warp_sum(den);
    Ltot = M == -INFINITY ? -INFINITY : M + log2f(den);
    for (int i = lane; i < np; i += 32) pw[i] = pl2[i] == -INFINITY ? 0.f : exp2f(pw[i] - Ltot);
  }
  __syncthreads();
  {
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < MPF; ++u) {
      const int i = r + RB * u;
      if (i < np) acc = fmaf(pw[i], opre[u], acc);
    }
    for (int i = r + RB * MPF; i < np; i += RB) acc = fmaf(pw[i], __ldcg(base + (size_t)i * (D + 2) + e), acc);
    float* rb = SC + 1024;      // [RB][D]
    rb[r * D + e] = acc;
    __syncthreads();
    if (tid < D) {
      float t = 0.f;
#pragma unroll
      for (int r2 = 0; r2 < RB; ++r2) t += rb[r2 * D + tid];
      out[((size_t)b * g.Hq + hq) * D + tid] = t;
    }
  }
  constexpr float kLn2 = 0.6931471805599453f;
  if (warp == 0) {
    if (lane == 0) {
      lse[(size_t)b * g.Hq + hq] = Ltot * kLn2;
      counters[(size_t)b * g.Hq + hq] = 0;
    }
    if (split_lse) {
      float* sl = split_lse + ((size_t)b * g.Hq + hq) * (ns + 1);
      for (int i = lane; i < ns; i += 32) sl[i] = pl2[2 * i] * kLn2;
      // the bf16 partial is the logsumexp of the CTAs' shares
      float Bm = -INFINITY;
      for (int i = lane; i < ns; i += 32) Bm = fmaxf(Bm, pl2[2 * i + 1]);
      Bm = warp_max(Bm);
      float Bs = 0.f;
      if (Bm != -INFINITY)
        for (int i = lane; i < ns; i += 32)
          if (pl2[2 * i + 1] != -INFINITY) Bs += exp2f(pl2[2 * i + 1] - Bm);
      Bs = warp_sum(Bs);
      if (lane == 0) sl[ns] = Bm == -INFINITY ? -INFINITY : (Bm + log2f(Bs)) * kLn2;
    }
  }
}

// Decode with one CTA per SM, each walking a contiguous, cost-balanced run of work items.  DBG
// and PM as for decode_kernel.  A CTA processes its items in order.  The producer warp runs ahead of the compute warps: it
// streams each item's code chunks through the ring (the next item's first chunks while the
// compute warps finish the current one), copies the step slices (the key slice when the KV head
// changes, the value slice per item) and computes the item's bf16 share.
// Every hand-off is an mbarrier whose phases both roles count the same way; every wait is
// bounded, and a wait that gives up sets the CTA's abort flag, after which neither role waits
// again (the items left are written as failed partials, so the merge counters stay exact).
template <int D, int C, bool DBG, int PM>
__global__ void __launch_bounds__(kThr, 1) decode_runs_kernel(
    Geo g, int layer, int step, int batch, const __nv_bfloat16* __restrict__ q,
    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ coded_len,
    const __nv_bfloat16* __restrict__ sink, const __nv_bfloat16* __restrict__ ring,
    const uint8_t* __restrict__ idx, const __nv_bfloat16* __restrict__ cbp, const float* __restrict__ rope, int ns,
    float* __restrict__ ws, float* __restrict__ out, float* __restrict__ lse, float* __restrict__ split_lse,
    int32_t* st) {
  using X = Dec<D, C>;
  const long wit = DBG ? g.wait_iters : kWaitIters;   // bound of every wait
  const bool pool = PM < 0 ? g.pool != 0 : PM != 0;
  constexpr int F = X::F, NG = X::NG, TQ = X::TQ, NPAIR = X::NPAIR, NREP = X::NREP;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* Ks = smem;
  const unsigned char* Vsm = smem + X::OFF_V;
  uint32_t* Hs = reinterpret_cast<uint32_t*>(smem + X::OFF_H);
  unsigned char* ringb = smem + X::OFF_RING;
  float2* zq = reinterpret_cast<float2*>(smem + X::OFF_ZQ);
  float2* etq_s = reinterpret_cast<float2*>(smem + X::OFF_TAB);       // [F] e^{-i TQ theta_f}
  float2* ech_s = etq_s + F;                                           // [F] e^{-i kChunk theta_f}
  float* red = reinterpret_cast<float*>(smem + X::OFF_RED);
  // misc: [0] abort, [1] merger, [2] chunks issued, [3] value slices issued, [5] key slices issued,
  // [6, 7] the CTA's item range
  int* misc = reinterpret_cast<int*>(smem + X::OFF_MISC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);
  float* SC = reinterpret_cast<float*>(smem + X::OFF_SC);    // scores, then weights; scratch elsewhere
  // bars[0]: key slice; bars[1]: value slice; bars[2 + s]: stage s full; bars[2 + kStages + s]:
  // stage s empty; bars[2 + 2 kStages]: "the item's slices are released" (compute warps, once per
  // item)
  const uint32_t bar_k = smem_addr(&bars[0]), bar_v = smem_addr(&bars[1]);
  const uint32_t bar_free = smem_addr(&bars[2 + 2 * kStages]);
  auto full_bar = [&](int gc) { return smem_addr(&bars[2 + gc % kStages]); };
  auto empty_bar = [&](int gc) { return smem_addr(&bars[2 + kStages + gc % kStages]); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool producer = warp == kCW;
  const int gq = g.Hq / g.H;
  const int blk = step / g.Tc, s = step % g.Tc;
  int32_t* counters = reinterpret_cast<int32_t*>(ws + (size_t)g.B * g.Hq * g.max_splits * 2 * (D + 2));
  auto slot_of = [&](const Item& x) { return ((size_t)x.b * g.Hq + x.hq) * g.max_splits * 2; };

  volatile int* abort_flag = misc;
  auto aborted = [&]() { return *abort_flag != 0; };
  // a bounded wait that gives up early once the CTA has aborted; on giving up it aborts the CTA
  auto wait_or_abort = [&](uint32_t bar, uint32_t parity) {
    if (aborted()) return false;
    for (long i = 0; i < wit; ++i) {
      if (mbar_wait(bar, parity, 1)) return true;
      if ((i & 63) == 63 && aborted()) return false;
    }
    *abort_flag = 1;
    return false;
  };

  if (tid == 0) {
    for (int i = 0; i < X::NBAR; ++i) mbar_init(smem_addr(&bars[i]), i >= 2 + kStages && i < 2 + 2 * kStages ? kCW : 1);
    fence_mbar_init();
    for (int i = 0; i < 8; ++i) misc[i] = 0;
  }
  __syncthreads();
  // Nothing is read before the programmatic-launch wait (the partition needs the counters).
  grid_dependency_wait();
  launch_dependents();
  if (warp == 0) {
    int a, z;
    partition_items(g, ctx_len, coded_len, batch, ns, blockIdx.x, gridDim.x, reinterpret_cast<unsigned char*>(SC),
                    a, z);
    if (lane == 0) {
      misc[6] = a;
      misc[7] = z;
    }
  }
  // position-independent RoPE steps of the score recurrence
  if (tid < F) {
    etq_s[tid] = cconj(rope_at(rope, g.RC, F, X::TQ, tid));
    ech_s[tid] = cconj(rope_at(rope, g.RC, F, kChunk, tid));
  }
  if (!producer)
    for (int i = tid; i < X::HB / 16; i += kCT) reinterpret_cast<uint4*>(Hs)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const int it0 = misc[6], it1 = misc[7];
  const float qscale = 1.4426950408889634f * rsqrtf((float)D);   // scores in log2 units

  if (producer) {
    // ==== producer warp
    int gc = 0;                        // ring position of the current item's first chunk
    int nv = 0, nk = 0, prev_h = -1;
    for (int it = it0, k = 0; it < it1; ++it, ++k) {
      const ItemGeo e = item_geo<D, C>(g, it, batch, ns, ctx_len, coded_len);
      const Item& x = e.x;
      const int n0 = e.sr.n0, n1 = e.sr.n1;
      constexpr int CPS = X::NSC / kChunk;           // chunks per full super-chunk
      // per-request streams: the K pages, then the V pages, of (layer, blk, b, h); pool mode: the
      // pools of (layer, blk, h), the request's pages found through the page table
      const uint8_t* kstream = idx + (pool ? idx_pool_off(g, layer, blk, x.h, 0) : idx_stream_off(g, layer, blk, x.b, x.h, 0));
      const uint8_t* vstream = idx + (pool ? idx_pool_off(g, layer, blk, x.h, 1) : idx_stream_off(g, layer, blk, x.b, x.h, 1));
      prefetch_share<D>(g, layer, step, x.b, x.h, x.j, ns, e.ctx, e.Lc, sink, ring, rope);
      if (lane == 0 && e.do_coded && k > 0) {
        // the compute warps' RoPE rows of the item's first chunk, into L2 ahead of them
        const int r0 = (g.S + n0) >> 3, r1 = (g.S + min(n1, n0 + kChunk) - 1) >> 3;
        prefetch_l2_bulk(rope + (size_t)r0 * F * 2, (uint32_t)(r1 - r0 + 1) * F * 8);
      }
      // first coded token, pages and K/V side of the item's chunk ci
      auto chunk_geom = [&](int ci, int& c0, int& np, bool& is_v) {
        const int sc = ci / (2 * CPS), r = ci % (2 * CPS);
        const int nkc = min(CPS, e.n_kchunks - sc * CPS);
        is_v = r >= nkc;
        c0 = n0 + (sc * CPS + (is_v ? r - nkc : r)) * kChunk;
        np = (min(n1, c0 + kChunk) - c0 + kPage - 1) / kPage;
      };
      // pool mode: the page ids of the next chunk to issue are loaded one chunk ahead (lane l holds
      // the chunk's pages l and l + 32) and range-checked only when they are used, so that the page
      // table's latency overlaps the ring's wait instead of stalling the producer
      int pf_ci = -1, pf_id[2] = {0, 0};
      const int32_t* pt_row = pool ? g.pt + (size_t)x.b * g.pts : nullptr;
      auto fetch_ids = [&](int ci) {
        int c0, np;
        bool v;
        chunk_geom(ci, c0, np, v);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = lane + 32 * hh;
          pf_id[hh] = i < np ? __ldg(pt_row + c0 / kPage + i) : 0;
        }
        pf_ci = ci;
      };
      // issue the item's chunk ci into ring position gc + ci.  Per-request streams: lane 0 alone,
      // one bulk copy of the chunk's pages.  Pool mode: the whole producer warp; lane l looks up the
      // chunk's pages l and l + 32 in the page table, and every run of consecutive physical pages
      // (within a half) is one bulk copy, issued by the lane at its start; an out-of-range entry is
      // reported and page 0 copied in its place (so that the stage still fills).
      auto issue_chunk = [&](int ci) {
        const int pos = gc + ci;
        if (lane == 0) misc[2] = pos + 1;
        if (DBG && (g.fault & kFaultDecodeDropChunk) && pos == 0) return;   // test hook: never issued
        int c0, np;
        bool is_v;
        chunk_geom(ci, c0, np, is_v);
        const uint32_t bar = full_bar(pos);
        const uint32_t dst = smem_addr(ringb + (pos % kStages) * X::STAGE);
        const uint8_t* src = is_v ? vstream : kstream;
        if (lane == 0) mbar_expect_tx(bar, np * X::PAGE);
        if (!pool) {
          bulk_g2s(dst, src + (size_t)(c0 / kPage) * X::PAGE, np * X::PAGE, bar);
          return;
        }
        if (pf_ci != ci) fetch_ids(ci);
        const int ids[2] = {pf_id[0], pf_id[1]};
        if (ci + 1 < e.n_stream) fetch_ids(ci + 1);     // in flight until the next chunk is issued
        __syncwarp();                                   // the expected bytes are set before any copy lands
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = lane + 32 * hh;                 // page of the chunk
          const int in_half = min(32, np - 32 * hh);    // pages of this half (may be <= 0)
          int id = i < np ? ids[hh] : 0;
          const bool bad = i < np && (id < 0 || id >= g.pool);
          if (bad) {
            set_status(st, LVQ_ECAPACITY);
            id = 0;
          }
          const int prev = __shfl_up_sync(0xffffffffu, id, 1);
          const bool prev_bad = __shfl_up_sync(0xffffffffu, bad, 1);
          const bool start = i < np && (lane == 0 || bad || prev_bad || id != prev + 1);
          const uint32_t starts = __ballot_sync(0xffffffffu, start);
          if (start) {
            const uint32_t later = lane < 31 ? starts >> (lane + 1) : 0u;
            const int end = later ? lane + __ffs(later) : in_half;   // lane of the next run's start
            bulk_g2s(dst + (uint32_t)i * X::PAGE, src + (size_t)id * X::PAGE, (uint32_t)(end - lane) * X::PAGE, bar);
          }
        }
      };
      // the ring is fed by lane 0 (per-request streams) or by the whole warp (pool mode): every chunk
      // whose stage its consumers have released, as lane 0 sees the stage
      int ci_next = 0;
      auto stage_free = [&](int ci) {
        const int pos = gc + ci;
        return pos < kStages || mbar_test(empty_bar(pos), (pos / kStages - 1) & 1);
      };
      auto service = [&]() {
        if (aborted()) return;
        if (pool) {
          while (ci_next < e.n_stream && __shfl_sync(0xffffffffu, lane == 0 ? (int)stage_free(ci_next) : 0, 0))
            issue_chunk(ci_next++);
        } else if (lane == 0) {
          while (ci_next < e.n_stream && stage_free(ci_next)) issue_chunk(ci_next++);
        }
      };
      bool to = aborted();
      // (1) the previous item is done with the step slices (a new KV head overwrites them); every
      // item's release is awaited, in order, so that the barrier's phases stay paired.  The ring
      // keeps being fed meanwhile.
      if (k > 0 && !to) {
        bool done = false;
        for (long i = 0; i < wit && !done; ++i) {
          done = __shfl_sync(0xffffffffu, lane == 0 ? (int)mbar_test(bar_free, (k - 1) & 1) : 0, 0) != 0;
          if (!done) {
            service();
            if ((i & 63) == 63 && __any_sync(0xffffffffu, aborted())) break;
          }
        }
        if (!done) {
          *abort_flag = 1;
          to = true;
        }
      }
      // (2) the step slices of a new KV head (they stay for the rest of its items)
      if (x.h != prev_h) {
        if (!to && lane == 0) {
          mbar_expect_tx(bar_k, X::KS);
          bulk_g2s(smem_addr(Ks), cbp + cbp_slice_off(g, layer, 0, blk, x.h, s), X::KS, bar_k);
          misc[5] = nk + 1;
          mbar_expect_tx(bar_v, X::KS);
          bulk_g2s(smem_addr(smem + X::OFF_V), cbp + cbp_slice_off(g, layer, 1, blk, x.h, s), X::KS, bar_v);
          misc[3] = nv + 1;
        }
        ++nk;
        ++nv;
        prev_h = x.h;
      }
      service();
      // (3) the rest of the item's chunks
      if (!to && (pool || lane == 0)) {
        for (; ci_next < e.n_stream; ++ci_next) {
          const int pos = gc + ci_next;
          bool ok = pos < kStages || wait_or_abort(empty_bar(pos), (pos / kStages - 1) & 1);
          if (pool) ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          issue_chunk(ci_next);
        }
      }
      gc += e.n_stream;
    }
  } else {
    // ==== compute warps
    int gc = 0;                        // ring position of the current item's first chunk
    int nk = 0, nv = 0, prev_h = -1;
    Lane<D, C> L;
    lane_init<D, C>(L, lane, etq_s);
    const int pi_own = L.vp / X::TPL, t_own = L.tq + TQ * (L.vp % X::TPL);   // the lane's token of a run
    const int gv = lane % NG, tp = lane / NG;
    const uint32_t hl = smem_addr(Hs) + (uint32_t)gv * 4;
    uint32_t* PW = reinterpret_cast<uint32_t*>(SC);
    for (int it = it0, k = 0; it < it1; ++it, ++k) {
      const ItemGeo e = item_geo<D, C>(g, it, batch, ns, ctx_len, coded_len);
      const Item& x = e.x;
      const int n0 = e.sr.n0, n1 = e.sr.n1;
      if (e.sr.bad && x.j == 0 && tid == 0) set_status(st, LVQ_ECAPACITY);
      bool timed_out = aborted();
      // a compute lane's RoPE factors at its first coded token
      float2 rf[X::CL];
      if (e.do_coded) {
        const int p_first = g.S + n0 + kPage * kPPW * warp + lane / X::NPV;
#pragma unroll
        for (int c2 = 0; c2 < X::CL; ++c2) rf[c2] = rope_at(rope, g.RC, F, p_first, L.f0 + c2);
      }
      // the query rotated to its own position, scaled so that scores come out in log2 units (the
      // previous item's readers of zq are past the barriers that ended it)
      if (tid < F && !e.sr.bad) {
        const __nv_bfloat16* qv = q + ((size_t)x.b * g.Hq + x.hq) * D;
        const float2 qraw = make_float2(__bfloat162float(qv[tid]), __bfloat162float(qv[tid + F]));
        const float2 qe = rope_at(rope, g.RC, F, e.ctx - 1, tid);
        zq[tid] = make_float2((qraw.x * qe.x - qraw.y * qe.y) * qscale, (qraw.y * qe.x + qraw.x * qe.y) * qscale);
      }
      // the item's bf16 share, by the compute warps (warp w takes tokens w, w + 15, ... straight from
      // global memory); the warps' partials are merged through the score array
      {
        compute_sync();                    // zq is complete
        float* part_bf16 = ws + (slot_of(x) + 2 * x.j + 1) * (D + 2);
        if (e.nbj > 0) {
          share_warp<D>(g, layer, step, x.b, x.h, x.j, ns, e.sr.S_eff, e.Lc, e.nbj, sink, ring, rope, zq, warp, kCW,
                        SC + warp * (D + 2));
          compute_sync();
          if (tid < D) {
            float M = -INFINITY;
#pragma unroll
            for (int w2 = 0; w2 < kCW; ++w2) M = fmaxf(M, SC[w2 * (D + 2) + D]);
            float o = 0.f, Ls = 0.f;
            if (M != -INFINITY)
#pragma unroll
              for (int w2 = 0; w2 < kCW; ++w2) {
                const float* pw2 = SC + w2 * (D + 2);
                if (pw2[D + 1] > 0.f) {
                  const float a = exp2f(pw2[D] - M);
                  o = fmaf(pw2[tid], a, o);
                  Ls = fmaf(pw2[D + 1], a, Ls);
                }
              }
            part_bf16[tid] = o;
            if (tid == 0) {
              part_bf16[D] = Ls > 0.f ? M : -INFINITY;
              part_bf16[D + 1] = Ls;
            }
          }
        } else if (tid < D + 2) {
          part_bf16[tid] = tid == D ? -INFINITY : 0.f;
        }
      }
      // the step slices of a new KV head (every one the producer copies is waited for, in order)
      if (x.h != prev_h) {
        if (!timed_out) timed_out = __any_sync(0xffffffffu, !wait_or_abort(bar_k, nk & 1));
        ++nk;
        if (!timed_out) timed_out = __any_sync(0xffffffffu, !wait_or_abort(bar_v, nv & 1));
        ++nv;
        prev_h = x.h;
      }
      compute_sync();
      float m_run = -INFINITY, l_run = 0.f;       // the coded partial, held by compute threads tid < NPAIR
      float2 o_run = make_float2(0.f, 0.f);
      if (e.do_coded) {
        float2 U[X::CL];                   // W of the lane's first token of the current chunk
#pragma unroll
        for (int c2 = 0; c2 < X::CL; ++c2) U[c2] = cmul(zq[L.f0 + c2], cconj(rf[c2]));
        int ci = 0;
        for (int sc = 0; sc < e.n_super; ++sc) {
          const int s0 = n0 + sc * X::NSC, s1 = min(n1, s0 + X::NSC);
          const int nkc = (s1 - s0 + kChunk - 1) / kChunk;
          // ---- phase A: scores of the super-chunk
          float mx = -INFINITY;
          for (int kc = 0; kc < nkc; ++kc, ++ci) {
            const int pos = gc + ci;
            if (!timed_out)
              timed_out = __any_sync(0xffffffffu, !wait_or_abort(full_bar(pos), (pos / kStages) & 1));
            if (!timed_out) {
              const int c0 = s0 + kc * kChunk;
              const unsigned char* stage = ringb + (pos % kStages) * X::STAGE;
              float2 Wc[X::CL], Wn[X::CL];
#pragma unroll
              for (int c2 = 0; c2 < X::CL; ++c2) {
                Wc[c2] = U[c2];
                Wn[c2] = cmul(U[c2], etq_s[L.f0 + c2]);        // s_1 = +1
              }
              // pages past the split's end hold stale codes: their tokens are masked
              const float sc_ = run_scores<D, C>(L, Ks, stage + warp * kPPW * X::PAGE, Wc, Wn);
              const int tok = c0 + kPage * (warp * kPPW + pi_own) + t_own;
              const float sv = tok < s1 ? sc_ : -INFINITY;
              mx = fmaxf(mx, sv);
              SC[tok - s0] = sv;
              __syncwarp();
              if (lane == 0) mbar_arrive(empty_bar(pos));
            }
#pragma unroll
            for (int c2 = 0; c2 < X::CL; ++c2) U[c2] = cmul(U[c2], ech_s[L.f0 + c2]);
          }
          // ---- weights: exact maximum, then integers round(2^(s - M) * 2^k) with 2^k * sum < 2^30
          mx = warp_max(mx);
          if (lane == 0) red[warp] = mx;
          timed_out = compute_sync_or(timed_out);
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kCW; ++w) M = fmaxf(M, red[w]);
          const int len = s1 - s0, len8 = (len + kPage - 1) & ~(kPage - 1);
          float ls = 0.f;
          if (!timed_out)
#pragma unroll 4
            for (int t = tid; t < len; t += kCT) {
              const float p = exp2f(SC[t] - M);
              SC[t] = p;
              ls += p;
            }
          ls = warp_sum(ls);
          if (lane == 0) red[16 + warp] = ls;
          compute_sync();
          float Ls = 0.f;
#pragma unroll
          for (int w = 0; w < kCW; ++w) Ls += red[16 + w];
          // Ls = m 2^E with m in [0.5, 1); Ls >= 1 (the maximum's weight is 1), so 17 <= 30 - E <= 29
          const int E = ((__float_as_int(Ls) >> 23) & 0xff) - 126;
          const int kfx = min(30, max(0, 30 - E));
          const float scale = __int_as_float((127 + kfx) << 23);
          uint32_t lf = 0;
          if (!timed_out)
#pragma unroll 4
            for (int t = tid; t < len8; t += kCT) {
              const uint32_t v = t < len ? __float2uint_rn(SC[t] * scale) : 0u;
              PW[t] = v;
              lf += v;
            }
          lf = warp_sum_u32(lf);
          if (lane == 0) reinterpret_cast<uint32_t*>(red)[32 + warp] = lf;
          compute_sync();
          uint32_t Lf = 0;
#pragma unroll
          for (int w = 0; w < kCW; ++w) Lf += reinterpret_cast<uint32_t*>(red)[32 + w];
          // ---- phase B: histogram of the weights over (code, group)
          for (int kc = 0; kc < nkc; ++kc, ++ci) {
            const int pos = gc + ci;
            if (!timed_out)
              timed_out = __any_sync(0xffffffffu, !wait_or_abort(full_bar(pos), (pos / kStages) & 1));
            if (timed_out) continue;
            const int c0 = s0 + kc * kChunk;
            const unsigned char* stage = ringb + (pos % kStages) * X::STAGE;
#pragma unroll 2
            for (int pi = 0; pi < kPPW; ++pi) {
              const int pl = warp * kPPW + pi;
              const int tb = c0 + kPage * pl;
              if (tb >= s1) break;
              hist_page<D, C>(stage + pl * X::PAGE + gv * kPage + tp * X::VPL, PW + (tb - s0) + tp * X::VPL, hl);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(pos));
          }
          timed_out = compute_sync_or(timed_out);
          // ---- contraction: o[ch] = sum_a H[a][ch / c] * V[a][ch], two channels per thread
          const int cp = tid % NPAIR, rep = tid / NPAIR;
          float2 acc = make_float2(0.f, 0.f);
          if (!timed_out && rep < NREP) {
            const uint32_t* vcol = reinterpret_cast<const uint32_t*>(Vsm) + cp;
            const uint32_t* hcol = Hs + (2 * cp) / C;
#pragma unroll 4
            for (int a = rep; a < kEntries; a += NREP) {
              const uint32_t v = vcol[a * NPAIR];
              const float hv = (float)hcol[a * NG];
              acc.x = fmaf(hv, bf16_lo(v), acc.x);
              acc.y = fmaf(hv, bf16_hi(v), acc.y);
            }
          }
          float2* rb = reinterpret_cast<float2*>(SC);      // [NREP][NPAIR]: the weights are no longer read
          if (rep < NREP) rb[rep * NPAIR + cp] = acc;
          compute_sync();
          if (tid < NPAIR && !timed_out && Lf > 0u) {
            float2 o = make_float2(0.f, 0.f);
#pragma unroll
            for (int r = 0; r < NREP; ++r) { o.x += rb[r * NPAIR + tid].x; o.y += rb[r * NPAIR + tid].y; }
            const float sc_scale = __int_as_float((127 - kfx) << 23);
            const float l_sc = (float)Lf * sc_scale;
            const float m_new = fmaxf(m_run, M);
            const float a_old = l_run > 0.f ? exp2f(m_run - m_new) : 0.f;
            const float a_new = exp2f(M - m_new) * sc_scale;
            o_run = make_float2(o_run.x * a_old + o.x * a_new, o_run.y * a_old + o.y * a_new);
            l_run = l_run * a_old + l_sc * exp2f(M - m_new);
            m_run = m_new;
          }
          // the histogram starts from zero for the next super-chunk or item
          for (int i = tid; i < X::HB / 16; i += kCT) reinterpret_cast<uint4*>(Hs)[i] = make_uint4(0u, 0u, 0u, 0u);
          compute_sync();
        }
      }
      gc += e.n_stream;
      // the item's slices are released (its last reads of Ks and Vsm are behind the barriers above)
      if (tid == 0) mbar_arrive(bar_free);
      // ---- the coded partial; the last item of this (request, head) to finish merges
      timed_out = timed_out || aborted();
      float* part_coded = ws + (slot_of(x) + 2 * x.j) * (D + 2);
      if (tid < NPAIR) {
        part_coded[2 * tid] = timed_out ? 0.f : o_run.x;
        part_coded[2 * tid + 1] = timed_out ? 0.f : o_run.y;
      }
      if (tid == 0) {
        part_coded[D] = timed_out || l_run == 0.f ? -INFINITY : m_run;
        part_coded[D + 1] = timed_out ? 0.f : l_run;
      }
      compute_sync();
      if (tid == 0) {
        __threadfence();                    // both partials (ordered before by the barriers) become visible
        misc[1] = atomicAdd(&counters[(size_t)x.b * g.Hq + x.hq], 1) == ns - 1;
      }
      compute_sync();
      if (misc[1])
        merge_partials<D>(ws, slot_of(x), ns, out + ((size_t)x.b * g.Hq + x.hq) * D, lse + (size_t)x.b * g.Hq + x.hq,
                               split_lse ? split_lse + ((size_t)x.b * g.Hq + x.hq) * (ns + 1) : nullptr,
                               &counters[(size_t)x.b * g.Hq + x.hq], SC);
    }
  }
  // every copy issued lands before the CTA exits
  if (__syncthreads_or(aborted())) {
    if (tid == 0) {
      set_status(st, LVQ_ETIMEOUT);
      if (misc[5] > 0) mbar_wait(bar_k, (misc[5] - 1) & 1, wit);
      if (misc[3] > 0) mbar_wait(bar_v, (misc[3] - 1) & 1, wit);
      for (int pos = max(0, misc[2] - kStages); pos < misc[2]; ++pos) mbar_wait(full_bar(pos), (pos / kStages) & 1, wit);
    }
    __syncthreads();
  }
}

template <int D, int C>
static cudaError_t decode_as(const Geo& g, int layer, int step, int batch, const __nv_bfloat16* q,
                             const int32_t* ctx_len, const int32_t* coded_len, const __nv_bfloat16* sink,
                             const __nv_bfloat16* ring, const uint8_t* idx, const __nv_bfloat16* cbp,
                             const float* rope, int ns, float* ws, float* out, float* lse,
                             float* split_lse, int32_t* st, cudaStream_t s) {
  static bool attr_set[kMaxDevices] = {};
  static int sm_count[kMaxDevices] = {};
  int dev = 0;
  cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return ge;
  int n_sm = 0;
  if (dev < 0 || dev >= kMaxDevices || !attr_set[dev]) {
    for (const void* fn : {(const void*)decode_kernel<D, C, false, 0>, (const void*)decode_kernel<D, C, false, 1>,
                           (const void*)decode_kernel<D, C, true, -1>, (const void*)decode_runs_kernel<D, C, false, 0>,
                           (const void*)decode_runs_kernel<D, C, false, 1>, (const void*)decode_runs_kernel<D, C, true, -1>}) {
      const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, Dec<D, C>::SMEM);
      if (e != cudaSuccess) return e;
    }
    const cudaError_t e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) {
      sm_count[dev] = n_sm;
      attr_set[dev] = true;
    }
  } else {
    n_sm = sm_count[dev];
  }
  // Work items: (request, query head, split).  One CTA per item (grid (ns, Hq, B)), unless the
  // caller caps the CTAs (lvq_decode_max_ctas) below the item count: then decode_runs_kernel, one
  // CTA per SM up to the cap, each walking a balanced run of items.  Its partition stages 16 bytes
  // per request in the score array (larger batches keep one CTA per item).
  const long long n_items = (long long)batch * g.Hq * ns;
  const int max_batch_runs = (Dec<D, C>::NSC * 4 - 8) / 16;
  const int cap = g.max_ctas > 0 && g.max_ctas < n_sm ? g.max_ctas : n_sm;
  const bool runs = g.max_ctas > 0 && n_items > cap && batch <= max_batch_runs;
  const bool dbg = g.fault != 0 || g.wait_iters != kWaitIters;   // the test hook is active
  cudaLaunchConfig_t lc = {};
  lc.gridDim = runs ? dim3(cap, 1, 1) : dim3(ns, g.Hq, batch);
  lc.blockDim = dim3(kThr, 1, 1);
  lc.dynamicSmemBytes = Dec<D, C>::SMEM;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may start during the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
#define LVQ_DEC_LAUNCH(DBGV, PMV)                                                                            \
  return runs ? cudaLaunchKernelEx(&lc, decode_runs_kernel<D, C, DBGV, PMV>, g, layer, step, batch, q, ctx_len,    \
                                   coded_len, sink, ring, idx, cbp, rope, ns, ws, out, lse, split_lse, st)         \
              : cudaLaunchKernelEx(&lc, decode_kernel<D, C, DBGV, PMV>, g, layer, step, q, ctx_len, coded_len, sink, \
                                   ring, idx, cbp, rope, ns, ws, out, lse, split_lse, st)
  if (dbg) LVQ_DEC_LAUNCH(true, -1);
  if (g.pool) LVQ_DEC_LAUNCH(false, 1);
  LVQ_DEC_LAUNCH(false, 0);
#undef LVQ_DEC_LAUNCH
}

// Sink + recent-window tokens one call can take: a CTA keeps the scores of its
// share of them in its score array (num_splits = 1 gives one CTA all of them).
template <int D, int C>
static int bf16_capacity_as() {
  return Dec<D, C>::NSC;
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
