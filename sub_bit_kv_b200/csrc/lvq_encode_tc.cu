// Prefill encoder on the 5th-generation tensor cores (tcgen05, TMEM).
//
// "LoopVQ summary", section "premises and limits": prefill keeps each step's
// keys and values until the last step, then computes the codebook distances
// with a matrix multiply and encodes.  Section "how it differs": the code is
// the single nearest entry of the joint vector.
//
// For a tile of 128 joint vectors X (one codebook) the tensor core computes
//   D[m][k] = ||C_k||^2 - 2 X_m . C_k          (k = 0..255)
// as one UMMA (M = 128, N = 256) whose K dimension holds the G vector
// elements and three extra columns: A = [X | 1 1 1 | 0...],
// B_k = [-2 C_k | n1 n2 n3 | 0...] with n1 + n2 + n3 = ||C_k||^2 split into
// bf16 parts.  bf16 products are exact and the tensor core accumulates in
// fp32 in TMEM.  ||X||^2 is left out: it does not change the argmin.
//
// Exactness: with eps = 2^-14 (||X||^2 + max_k ||C_k||^2), every entry whose
// exact distance is the minimum has D <= min(D) + eps.  The epilogue finds
// min(D), then the set of entries with D <= min(D) + eps.  A single candidate
// is the exact nearest entry; several (a near-tie) are rescored in fp64 in the
// direct form sum_j (X_j - C_kj)^2 -- exact for bf16 inputs -- lowest index on
// ties.  So every code equals the fp64 brute-force answer.
//
// One persistent CTA per SM (it allocates all 512 TMEM columns), warp-specialised:
//  * warp 9 (one lane) streams raw input tiles [Tc][128 tokens][16 channels] by
//    TMA (no multicast) into a 3-stage ring (full/empty mbarriers);
//  * warp 8 (one lane) issues the UMMAs: group-tile k of an item goes to
//    accumulator k % 2 (256 TMEM columns each) once its A tile is ready and the
//    accumulator's previous contents have been read, and commits to that
//    accumulator's "full" barrier;
//  * warps 0-3 (team 0) and 4-7 (team 1) each own one accumulator and take every
//    other group-tile; thread r of a team owns row r (TMEM lane r, one token).
//    For the team's next group-tile it builds row r of the A tile from the raw
//    tile (and the row's ||x||^2), then drains the current accumulator: all 256
//    columns of its row in four 64-column loads, the accumulator released to the
//    MMA warp as soon as the last load has landed.  Per 32-column block it keeps
//    the block minimum (3-input min) and the block's columns within eps of it as
//    a bit mask, made on the FMA pipe: with 2^k scaled so that any fp32 value
//    below the threshold t gives (t - v) 2^k >= 1, a saturating FMA turns each
//    column into an exact 0 or 1 and a packed FMA shifts them into two float
//    accumulators (even and odd columns).  The row's code follows from its eight
//    block minima and masks, with fp64 rescoring of near-ties.
// Work items are (K/V, block, head, 16-channel span) x 8192-token ranges; the
// item's B tiles (its 16/c codebooks) are rebuilt between items.
#include "lvq_common.cuh"

namespace lvq {

namespace tc {

constexpr int kTeamWarps = 4;                    // one accumulator per team, one row per thread
constexpr int kMmaWarp = 2 * kTeamWarps;         // warp 8: UMMA issue
constexpr int kTmaWarp = kMmaWarp + 1;           // warp 9: raw-tile TMA
constexpr int kThreads = 32 * (kTmaWarp + 1);    // 320
constexpr int kRows = 128;                       // UMMA M
constexpr int kTileTokens = 128;
constexpr int kItemTokens = 8192;                // tokens per work item (64 tiles)
constexpr int kSpan = 16;                        // channels per item (TMA box x: 32 bytes)
constexpr int kRawStages = 3;
constexpr int kBlocks = kEntries / 32;           // 32-column blocks of a row

template <int G, int C>
struct Enc {
  static constexpr int TC = G / C;            // steps per block
  static constexpr int NGC = kSpan / C;       // groups per item (even: the teams alternate)
  static constexpr int KP = G + 16;           // padded K: G elements, 3 bias columns, zeros
  static constexpr int KSTEPS = KP / 16;
  static constexpr int SBO = KP * 16;         // bytes between 8-row core-matrix groups
  static constexpr int A_TILE = kRows * KP * 2;
  static constexpr int B_TILE = kEntries * KP * 2;
  static constexpr int RAW = TC * kTileTokens * kSpan * 2;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_A = OFF_B + NGC * B_TILE;                // [team][slot]
  static constexpr int OFF_RAW = OFF_A + 4 * A_TILE;
  static constexpr int OFF_NMAX = OFF_RAW + kRawStages * RAW;
  static constexpr int OFF_BAR = OFF_NMAX + 64;
  static constexpr int NBAR = 2 * kRawStages + 4 + 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;                 // + alignment slack
  static_assert(NGC == 2 || NGC == 4, "two teams alternate over the item's groups");
  static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");
  static_assert(KP % 16 == 0 && G % 8 == 0, "K steps, 16-byte chunks of a row");
};

// K-major, no-swizzle UMMA shared-memory descriptor: core matrices of 8 rows x
// 16 bytes, the two K-adjacent core matrices LBO = 128 bytes apart, 8-row
// groups SBO bytes apart; version 1 (sm_100).
__device__ inline uint64_t smem_desc(uint32_t addr, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3fff) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46);
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

// byte offset of element (row, k) of a K-major no-swizzle tile
__device__ inline uint32_t kmaj_off(int row, int k, int sbo) {
  return (row & 7) * 16 + (row >> 3) * sbo + (k >> 3) * 128 + (k & 7) * 2;
}

// byte offset of channel ch of token row r (of step s) in a raw tile written by TMA with
// the 32-byte swizzle: each token row is 32 bytes, and its two 16-byte halves trade
// places when bit 2 of r is set (address bit 4 ^= bit 7), so that eight consecutive
// rows' 16-byte halves fall in distinct bank groups
__device__ inline uint32_t raw_off(int s, int r, int ch) {
  return (uint32_t)((s * kTileTokens + r) * 32 + ((((ch >> 3) ^ (r >> 2)) & 1) << 4) + (ch & 7) * 2);
}

__device__ inline void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ inline void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ inline void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void mbar_arrive1(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

__device__ inline void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      :: "r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc) : "memory");
}

__device__ inline void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar)
               : "memory");
}

// 64 consecutive fp32 columns of this thread's TMEM lane, issued without waiting
// (tcgen05.wait::ld completes every load issued before it)
__device__ inline void tmem_ld64_nowait(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,"
      "%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}
__device__ inline void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ inline float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ inline float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Candidate masks use a permuted bit order: column 2p of a block is bit 31 - p,
// column 2p + 1 is bit 15 - p.  Column of mask bit b:
__device__ inline int mask_col(int b) { return b >= 16 ? 2 * (31 - b) : 2 * (15 - b) + 1; }

// Four 32-column blocks of a row (columns 0-31 and 32-63 of `ra`, then of `rb`), processed
// in lockstep so that their chains overlap: each block's minimum bm[b], and its columns
// v < bm[b] + eps as a bit mask in the permuted order above.  eps > 0 is at least
// 2^-15 |bm| (so bm + eps > bm).
__device__ inline void quad_min_mask(const uint32_t (&ra)[64], const uint32_t (&rb)[64], float eps, float (&bm)[4],
                                     uint32_t (&mask)[4]) {
  // column i of block b (both compile-time after unrolling: the arrays stay in registers)
  auto V = [&](int b, int i) -> float { return __uint_as_float(b < 2 ? ra[32 * b + i] : rb[32 * (b - 2) + i]); };
  float m[4][4];
#pragma unroll
  for (int b = 0; b < 4; ++b)
#pragma unroll
    for (int u = 0; u < 4; ++u) m[b][u] = V(b, u);
#pragma unroll
  for (int i = 4; i < 28; i += 8)        // columns 4..27: four chains per block, two columns a step
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int u = 0; u < 4; ++u)
        m[b][u] = fmin3(m[b][u], V(b, i + 2 * u), V(b, i + 2 * u + 1));
#pragma unroll
  for (int b = 0; b < 4; ++b) {          // columns 28..31
    const float a0 = fmin3(m[b][0], V(b, 28), V(b, 29));
    const float a1 = fmin3(m[b][1], V(b, 30), V(b, 31));
    bm[b] = fminf(fmin3(a0, a1, m[b][2]), m[b][3]);
  }
  // Any fp32 v < tb lies at least 2^(e-24) below it (e the exponent of tb), so with
  // k = 24 - e, (tb - v) 2^k >= 1 and sat(fma(v, -2^k, tb 2^k)) is exactly 1; any v >= tb
  // gives exactly 0 (an overflow to infinity keeps the sign, so it saturates the same way).
  float tb[4], nsc[4], c[4];
  bool fast = true;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    tb[b] = bm[b] + eps;
    const uint32_t E = (__float_as_uint(tb[b]) >> 23) & 0xffu;   // biased exponent of tb
    fast = fast && E >= 24u;
    const float sc = __uint_as_float((278u - (E < 24u ? 24u : E)) << 23);   // 2^k, k = 151 - E
    nsc[b] = -sc;
    c[b] = tb[b] * sc;                                         // exact: a power-of-two scale
  }
  if (fast) {
    // per block two accumulators (pairs 0-7 and 8-15) of s = 0/1 shifted in: exact integers
    float2 lo[4], hi[4];
    const float2 two = make_float2(2.f, 2.f);
#pragma unroll
    for (int b = 0; b < 4; ++b) lo[b] = hi[b] = make_float2(0.f, 0.f);
#pragma unroll
    for (int p = 0; p < 8; ++p)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float s0 = fma_sat(V(b, 2 * p), nsc[b], c[b]);
        const float s1 = fma_sat(V(b, 2 * p + 1), nsc[b], c[b]);
        const float s2 = fma_sat(V(b, 2 * p + 16), nsc[b], c[b]);
        const float s3 = fma_sat(V(b, 2 * p + 17), nsc[b], c[b]);
        lo[b] = __ffma2_rn(lo[b], two, make_float2(s0, s1));
        hi[b] = __ffma2_rn(hi[b], two, make_float2(s2, s3));
      }
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      // 16-bit integers (pair 0 on top), plus 2^23 so that they sit in the low mantissa bits
      const float2 m2 = __ffma2_rn(lo[b], make_float2(256.f, 256.f), hi[b]);
      const float2 w = __fadd2_rn(m2, make_float2(8388608.f, 8388608.f));
      mask[b] = __byte_perm(__float_as_uint(w.y), __float_as_uint(w.x), 0x5410);
    }
  } else {
    // some tb is zero, subnormal or tiny: compare the plain way (sign of tb - v per column)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      uint32_t sa = 0u, sb = 0u;
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        sa = (sa << 1) | (tb[b] - V(b, 2 * p) > 0.f ? 1u : 0u);
        sb = (sb << 1) | (tb[b] - V(b, 2 * p + 1) > 0.f ? 1u : 0u);
      }
      mask[b] = (sa << 16) | sb;
    }
  }
}

template <int G, int C>
__global__ void __launch_bounds__(kThreads, 1) encode_tc_kernel(
    const __grid_constant__ CUtensorMap tmap, Geo g, int layer0, int n_layers, int req, int tok_begin, int n_tok,
    int coded_offset, const __nv_bfloat16* __restrict__ cb, uint8_t* __restrict__ idx, int32_t* st) {
  using X = Enc<G, C>;
  constexpr int TC = X::TC, NGC = X::NGC, SBO = X::SBO;
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte alignment of the dynamic shared memory base
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* Bt = smem + X::OFF_B;
  unsigned char* At = smem + X::OFF_A;
  unsigned char* raw = smem + X::OFF_RAW;
  float* nmax_s = reinterpret_cast<float*>(smem + X::OFF_NMAX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);
  // bars: [0, NR) raw full, [NR, 2NR) raw empty, then A ready [team][slot], acc full [team], acc empty [team]
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = bars + kRawStages;
  uint64_t* a_ready = bars + 2 * kRawStages;
  uint64_t* acc_full = a_ready + 4;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + X::OFF_MISC);
  volatile int* fail_s = reinterpret_cast<volatile int*>(smem + X::OFF_MISC + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int team = warp / kTeamWarps;     // 0, 1 (2 for the MMA and TMA warps)
  const int row = tid & (kRows - 1);      // TMEM lane = tile row = token of the tile (team warps)

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" :: "r"(smem_addr(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kRawStages; ++i) {
      mbar_init(smem_addr(&raw_full[i]), 1);
      mbar_init(smem_addr(&raw_empty[i]), 2 * kTeamWarps);
    }
    for (int i = 0; i < 4; ++i) mbar_init(smem_addr(&a_ready[i]), kTeamWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&acc_full[i]), 1);
      mbar_init(smem_addr(&acc_empty[i]), kTeamWarps);
    }
    fence_mbar_init();
    *fail_s = 0;
  }
  // A tiles: [x | 1 1 1 | 0...]; the columns from G on never change
  for (int i = tid; i < 4 * X::A_TILE / 16; i += kThreads) {
    const int a = i / (X::A_TILE / 16), rem = i % (X::A_TILE / 16);
    const int r = rem / (X::KP / 8), k8 = rem % (X::KP / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (k8 * 8 == G) v = make_uint4(0x3f803f80u, 0x3f80u, 0u, 0u);   // bf16 1.0 in columns G .. G+2
    *reinterpret_cast<uint4*>(At + a * X::A_TILE + kmaj_off(r, k8 * 8, SBO)) = v;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long wit = g.wait_iters;

  const int n_spans = g.d / kSpan;
  const int n_sets = 2 * g.nblk * g.H * n_spans;
  const int n_ranges = (n_tok + kItemTokens - 1) / kItemTokens;
  const long n_items = (long)n_sets * n_ranges * n_layers;    // layers outermost

  long T_glob = 0;          // raw tiles of the items before this one (this CTA)
  long J_glob = 0;          // group-tiles per team of the items before this one
  // in-flight bookkeeping for a failed run: the last MMA issued per accumulator, tiles issued
  long last_mma[2] = {-1, -1};
  long tiles_issued = 0;

  for (long item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int lrel = (int)(item / ((long)n_sets * n_ranges));   // layer layer0 + lrel
    const int layer = layer0 + lrel;
    int cs = (int)(item % ((long)n_sets * n_ranges) / n_ranges);
    const int range = (int)(item % n_ranges);
    const int span = cs % n_spans; cs /= n_spans;
    const int h = cs % g.H; cs /= g.H;
    const int blk = cs % g.nblk; cs /= g.nblk;
    const int kvi = cs;
    const int t_first = tok_begin + range * kItemTokens;
    const int t_last = min(tok_begin + n_tok, t_first + kItemTokens);
    const int n_tiles = (t_last - t_first + kTileTokens - 1) / kTileTokens;
    const int n_j = n_tiles * NGC / 2;              // group-tiles per team

    // every role has finished the previous item: its MMAs completed (the teams waited for
    // each), its raw tiles landed (the teams waited for each)
    __syncthreads();
    if (*fail_s) break;
    if (tid < NGC) nmax_s[tid] = 0.f;
    __syncthreads();
    // B tiles: [-2 C_k | n1 n2 n3 | 0] for the item's groups, K-major no-swizzle;
    // nmax_s[gi] = max_k ||C_k||^2 (non-negative floats order like their bits)
    for (int e = tid; e < NGC * kEntries; e += kThreads) {
      const int gi = e / kEntries, k = e % kEntries;
      const int grp = span * NGC + gi;
      const uint4* ce = reinterpret_cast<const uint4*>(cb + cb_off(g, layer, kvi, blk, h, grp) + (size_t)k * G);
      unsigned char* bt = Bt + gi * X::B_TILE;
      double n = 0.0;
#pragma unroll
      for (int j8 = 0; j8 < G / 8; ++j8) {
        const uint4 w = __ldg(ce + j8);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = bf16_lo(ww[q]), hi = bf16_hi(ww[q]);
          n = fma((double)lo, (double)lo, n);
          n = fma((double)hi, (double)hi, n);
          const __nv_bfloat162 m2 = __floats2bfloat162_rn(-2.f * lo, -2.f * hi);   // exact
          o[q] = *reinterpret_cast<const uint32_t*>(&m2);
        }
        *reinterpret_cast<uint4*>(bt + kmaj_off(k, j8 * 8, SBO)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      const __nv_bfloat16 n1 = __double2bfloat16(n);
      const double r1 = n - (double)__bfloat162float(n1);
      const __nv_bfloat16 n2 = __double2bfloat16(r1);
      const __nv_bfloat16 n3 = __double2bfloat16(r1 - (double)__bfloat162float(n2));
      *reinterpret_cast<uint4*>(bt + kmaj_off(k, G, SBO)) =
          make_uint4((uint32_t)__bfloat16_as_ushort(n1) | ((uint32_t)__bfloat16_as_ushort(n2) << 16),
                     (uint32_t)__bfloat16_as_ushort(n3), 0u, 0u);
      *reinterpret_cast<uint4*>(bt + kmaj_off(k, G + 8, SBO)) = make_uint4(0u, 0u, 0u, 0u);
      atomicMax(reinterpret_cast<int*>(&nmax_s[gi]), __float_as_int((float)n));
    }
    fence_proxy_async();
    __syncthreads();

    if (warp == kTmaWarp) {
      // ---- raw tiles of the item, through the ring
      if (lane == 0) {
        for (int t = 0; t < n_tiles; ++t) {
          const long T = T_glob + t;
          const int stg = (int)(T % kRawStages);
          if (T >= kRawStages &&
              (*fail_s || !mbar_wait_sleep(smem_addr(&raw_empty[stg]), (uint32_t)((T / kRawStages - 1) & 1), wit))) {
            *fail_s = 1;
            break;
          }
          const uint32_t bar = smem_addr(&raw_full[stg]);
          mbar_expect_tx(bar, X::RAW);
          tma_load_3d(smem_addr(raw + stg * X::RAW), &tmap, h * g.d + span * kSpan, t_first + t * kTileTokens,
                      (lrel * 2 + kvi) * g.T + blk * TC, bar);
          tiles_issued = T + 1;
        }
      }
    } else if (warp == kMmaWarp) {
      // ---- UMMAs: group-tile k of the item goes to accumulator k % 2
      if (lane == 0) {
        for (int k = 0; k < n_tiles * NGC; ++k) {
          const int tm = k & 1;
          const long J = J_glob + (k >> 1);
          const int slot = (int)(J & 1);
          if (*fail_s || !mbar_wait_sleep(smem_addr(&a_ready[tm * 2 + slot]), (uint32_t)((J >> 1) & 1), wit) ||
              (J >= 1 && !mbar_wait_sleep(smem_addr(&acc_empty[tm]), (uint32_t)((J - 1) & 1), wit))) {
            *fail_s = 1;
            break;
          }
          tc_fence_after();
          const int gi = k % NGC;
          const uint32_t a0 = smem_addr(At + (tm * 2 + slot) * X::A_TILE), b0 = smem_addr(Bt + gi * X::B_TILE);
#pragma unroll
          for (int ks = 0; ks < X::KSTEPS; ++ks)
            mma_bf16(tmem_base + (uint32_t)(tm * 256), smem_desc(a0 + ks * 256, SBO), smem_desc(b0 + ks * 256, SBO),
                     kIdesc, ks > 0);
          mma_commit(smem_addr(&acc_full[tm]));
          last_mma[tm] = J;
        }
      }
    } else {
      // ---- a team: group-tiles j = 0, 1, ... of the item are k = 2 j + team
      const uint32_t tmem_acc = tmem_base + (uint32_t)(team * 256) + ((uint32_t)(32 * (warp & 3)) << 16);
      // builds row `row` of the A tile of team group-tile j; returns ||x||^2 of the row, or a
      // negative value if a wait timed out (uniform over the warp)
      auto build = [&](int j) -> float {
        const int k = 2 * j + team, t = k / NGC, gi = k % NGC;
        const long T = T_glob + t, J = J_glob + j;
        const int stg = (int)(T % kRawStages);
        const bool ok = !*fail_s && mbar_wait_sleep(smem_addr(&raw_full[stg]), (uint32_t)((T / kRawStages) & 1), wit);
        if (__any_sync(0xffffffffu, !ok)) return -1.f;
        const unsigned char* rw = raw + stg * X::RAW;
        unsigned char* at = At + (team * 2 + (int)(J & 1)) * X::A_TILE;
        uint32_t xw[G / 2];
#pragma unroll
        for (int s2 = 0; s2 < TC; ++s2) {
          const unsigned char* src = rw + raw_off(s2, row, gi * C);
          if constexpr (C == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(src);
            xw[s2 * 2] = w.x;
            xw[s2 * 2 + 1] = w.y;
          } else {
            const uint4 w = *reinterpret_cast<const uint4*>(src);
            xw[s2 * 4] = w.x;
            xw[s2 * 4 + 1] = w.y;
            xw[s2 * 4 + 2] = w.z;
            xw[s2 * 4 + 3] = w.w;
          }
        }
        float2 x2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < G / 2; ++q) {
          const float2 v = make_float2(bf16_lo(xw[q]), bf16_hi(xw[q]));
          x2 = __ffma2_rn(v, v, x2);
        }
#pragma unroll
        for (int c8 = 0; c8 < G / 8; ++c8)
          *reinterpret_cast<uint4*>(at + kmaj_off(row, c8 * 8, SBO)) =
              make_uint4(xw[c8 * 4], xw[c8 * 4 + 1], xw[c8 * 4 + 2], xw[c8 * 4 + 3]);
        fence_proxy_async();             // the tile is read by the tensor core (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive1(smem_addr(&a_ready[team * 2 + (int)(J & 1)]));
        return x2.x + x2.y;
      };
      float xx_cur = n_j > 0 ? build(0) : 0.f;
      bool ok = xx_cur >= 0.f;
      for (int j = 0; j < n_j && ok; ++j) {
        const int k = 2 * j + team, t = k / NGC, gi = k % NGC;
        const long J = J_glob + j, T = T_glob + t;
        const int stg = (int)(T % kRawStages);
        float xx_next = 0.f;
        if (j + 1 < n_j) {
          xx_next = build(j + 1);
          ok = xx_next >= 0.f;
        }
        if (ok) ok = !*fail_s && mbar_wait_sleep(smem_addr(&acc_full[team]), (uint32_t)(J & 1), wit);
        if (__any_sync(0xffffffffu, !ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // eps = 2^-14 (||x||^2 + max ||C||^2), at least 2^-120 so that bm + eps > bm always
        const float eps = fmaxf((xx_cur + nmax_s[gi]) * 0x1p-14f, 0x1p-120f);
        float bmin[kBlocks];
        uint32_t mask[kBlocks];
        {
          uint32_t ra[64], rb[64];
          tmem_ld64_nowait(tmem_acc + 0, ra);
          tmem_ld64_nowait(tmem_acc + 64, rb);
          tmem_wait_ld();
          float q0[4], q1[4];
          uint32_t k0[4], k1[4];
          quad_min_mask(ra, rb, eps, q0, k0);
          tmem_ld64_nowait(tmem_acc + 128, ra);
          tmem_ld64_nowait(tmem_acc + 192, rb);
          tmem_wait_ld();
          // every column of the row is in registers: the accumulator may be overwritten
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive1(smem_addr(&acc_empty[team]));
          quad_min_mask(ra, rb, eps, q1, k1);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            bmin[b] = q0[b];
            bmin[4 + b] = q1[b];
            mask[b] = k0[b];
            mask[4 + b] = k1[b];
          }
        }
        const float mrow = fminf(fmin3(bmin[0], bmin[1], bmin[2]), fmin3(bmin[3], bmin[4], fmin3(bmin[5], bmin[6], bmin[7])));
        const float thr = mrow + eps;
        uint32_t bmask = 0, at_min = 0;   // blocks that can hold a candidate / that hold the minimum
#pragma unroll
        for (int q = 0; q < kBlocks; ++q) {
          bmask |= bmin[q] <= thr ? 1u << q : 0u;
          at_min |= bmin[q] == mrow ? 1u << q : 0u;
        }
        const int wb = __ffs(at_min) - 1;               // the first block holding the minimum
        // mask[wb] by a three-level select on the bits of wb
        const uint32_t c01 = wb & 1 ? mask[1] : mask[0], c23 = wb & 1 ? mask[3] : mask[2];
        const uint32_t c45 = wb & 1 ? mask[5] : mask[4], c67 = wb & 1 ? mask[7] : mask[6];
        const uint32_t c03 = wb & 2 ? c23 : c01, c47 = wb & 2 ? c67 : c45;
        const uint32_t cm = wb & 4 ? c47 : c03;
        const int t0 = t_first + t * kTileTokens;
        if (t0 + row < t_last) {
          int code = wb * 32 + mask_col(31 - __clz(cm));
          if (__popc(cm) + __popc(bmask & ~(1u << wb)) > 1) {
            // near-tie: exact fp64 direct-form distances of the candidates of every block within
            // eps (the block masks are supersets of them), lowest index on ties
            const unsigned char* bt = Bt + gi * X::B_TILE;
            const unsigned char* rw = raw + stg * X::RAW;
            float xf[G];                                    // the row's joint vector, element s*c + e
#pragma unroll
            for (int s2 = 0; s2 < TC; ++s2)
#pragma unroll
              for (int e = 0; e < C; ++e)
                xf[s2 * C + e] = __bfloat162float(
                    *reinterpret_cast<const __nv_bfloat16*>(rw + raw_off(s2, row, gi * C + e)));
            double best = 1e300;
            int bk = kEntries;
#pragma unroll 1
            for (int q = 0; q < kBlocks; ++q) {
              if (!((bmask >> q) & 1u)) continue;
              for (uint32_t m = mask[q]; m; m &= m - 1u) {
                const int kk = q * 32 + mask_col(__ffs(m) - 1);
                // sum_j (x_j - C_kj)^2 in two chains; the tile holds -2 C (exact halving)
                double d2a = 0.0, d2b = 0.0;
#pragma unroll
                for (int j8 = 0; j8 < G / 8; ++j8) {
                  const uint4 cw = *reinterpret_cast<const uint4*>(bt + kmaj_off(kk, j8 * 8, SBO));
                  const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                  for (int q2 = 0; q2 < 4; ++q2) {
                    const double da = (double)xf[j8 * 8 + 2 * q2] + 0.5 * (double)bf16_lo(w4[q2]);
                    const double db = (double)xf[j8 * 8 + 2 * q2 + 1] + 0.5 * (double)bf16_hi(w4[q2]);
                    d2a = fma(da, da, d2a);
                    d2b = fma(db, db, d2b);
                  }
                }
                const double d2 = d2a + d2b;
                if (d2 < best || (d2 == best && kk < bk)) { best = d2; bk = kk; }
              }
            }
            code = bk;
          }
          const int cn = coded_offset + (t0 + row - tok_begin);
          const int phys = phys_page(g, req, cn >> 3);
          if (phys >= 0)
            idx[idx_code_off(g, layer, blk, req, h, kvi, phys, cn, span * NGC + gi)] = (uint8_t)code;
          else
            set_status(st, LVQ_ECAPACITY);
        }
        // the last group-tile of raw tile t for this team: the stage may be refilled
        if (gi + 2 >= NGC) {
          __syncwarp();
          if (lane == 0) mbar_arrive1(smem_addr(&raw_empty[stg]));
        }
        xx_cur = xx_next;
      }
      if (!ok && lane == 0) *fail_s = 1;
    }
    T_glob += n_tiles;
    J_glob += n_j;
  }
  __syncthreads();
  const bool failed = *fail_s != 0;
  if (failed) {
    if (tid == 0) set_status(st, LVQ_ETIMEOUT);
    // let every issued MMA and tile copy finish before TMEM and shared memory are released
    if (warp == kMmaWarp && lane == 0)
      for (int tm = 0; tm < 2; ++tm)
        if (last_mma[tm] >= 0) mbar_wait(smem_addr(&acc_full[tm]), (uint32_t)(last_mma[tm] & 1), wit);
    if (warp == kTmaWarp && lane == 0)
      for (long T = tiles_issued - kRawStages; T < tiles_issued; ++T)
        if (T >= 0) mbar_wait(smem_addr(&raw_full[T % kRawStages]), (uint32_t)((T / kRawStages) & 1), wit);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" :: "r"(tmem_base) : "memory");
}

}  // namespace tc

// (G, c) = (32, 4) would need Tc = 8 raw steps per tile: its shared-memory plan does not fit one
// CTA, so the direct-form encoder serves it
bool encode_tc_supported(int G, int c) { return (G == 16 && (c == 4 || c == 8)) || (G == 32 && c == 8); }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda dependency)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

template <int G, int C>
static cudaError_t encode_tc_as(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                                int kv_tokens, int tok_begin, int n_tok, int coded_offset,
                                const __nv_bfloat16* cb, uint8_t* idx, int32_t* st, cudaStream_t s) {
  using X = tc::Enc<G, C>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  // layer < 0: every layer in one launch; kv then holds the layers back to back
  const int layer0 = layer < 0 ? 0 : layer, n_layers = layer < 0 ? g.L : 1;
  CUtensorMap map;
  // dims: channels of a token row (H*d), tokens, (layer, kv, step) planes
  cuuint64_t dims[3] = {(cuuint64_t)g.H * g.d, (cuuint64_t)kv_tokens, (cuuint64_t)n_layers * 2 * g.T};
  cuuint64_t strides[2] = {(cuuint64_t)tok_stride * 2, (cuuint64_t)tok_stride * kv_tokens * 2};
  cuuint32_t box[3] = {tc::kSpan, tc::kTileTokens, (cuuint32_t)X::TC};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(kv), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

  static bool attr_set[kMaxDevices] = {};
  static int n_sm[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(tc::encode_tc_kernel<G, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, X::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const long n_sets = 2L * g.nblk * g.H * (g.d / tc::kSpan);
  const long items = n_sets * ((n_tok + tc::kItemTokens - 1) / tc::kItemTokens) * n_layers;
  const int grid = (int)std::min<long>(items, n_sm[dev]);
  tc::encode_tc_kernel<G, C><<<grid, tc::kThreads, X::SMEM, s>>>(map, g, layer0, n_layers, req, tok_begin, n_tok,
                                                                  coded_offset, cb, idx, st);
  return cudaGetLastError();
}

cudaError_t launch_encode_tc(const Geo& g, int layer, int req, const __nv_bfloat16* kv, int64_t tok_stride,
                             int kv_tokens, int tok_begin, int n_tok, int coded_offset,
                             const __nv_bfloat16* cb, uint8_t* idx, int32_t* st, cudaStream_t s) {
  if (n_tok == 0) return cudaSuccess;
#define LVQ_ETC(GG, CC)                                                                                  \
  if (g.G == GG && g.c == CC)                                                                            \
    return encode_tc_as<GG, CC>(g, layer, req, kv, tok_stride, kv_tokens, tok_begin, n_tok, coded_offset, \
                                cb, idx, st, s);
  LVQ_ETC(16, 4) LVQ_ETC(16, 8) LVQ_ETC(32, 8)
#undef LVQ_ETC
  return cudaErrorInvalidValue;
}

}  // namespace lvq
