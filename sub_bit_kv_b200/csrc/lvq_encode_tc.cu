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
// CTA: 512 threads, one per SM (it allocates all 512 TMEM columns).  Work items
// are (K/V, block, head, 16-channel span) x 1024-token ranges.  The raw input
// tile [Tc][128 tokens][16 channels] arrives by TMA (no multicast) into a
// 2-stage ring; the 16 channels hold 16/c groups.  Two sets of 8 warps each own
// 256 TMEM columns and alternate over the groups: build the group's A tile,
// issue its UMMA, and run the argmin epilogue, so one set's epilogue overlaps
// the other set's MMA.  In a set, warps w and w + 4 read the same TMEM lane
// quadrant (32 rows) and split the 256 entries into halves.
#include "lvq_common.cuh"

namespace lvq {

namespace tc {

constexpr int kThreads = 512;
constexpr int kSetThreads = 256;    // one MMA set: 8 warps
constexpr int kRows = 128;          // UMMA M
constexpr int kTileTokens = 128;
constexpr int kItemTokens = 1024;   // tokens per work item (8 tiles)
constexpr int kSpan = 16;           // channels per item (TMA box x: 32 bytes)
constexpr int kRawStages = 2;

template <int G, int C>
struct Enc {
  static constexpr int TC = G / C;            // steps per block
  static constexpr int NGC = kSpan / C;       // groups per item
  static constexpr int KP = G + 16;           // padded K: G elements, 3 bias columns, zeros
  static constexpr int KSTEPS = KP / 16;
  static constexpr int SBO = KP * 16;         // bytes between 8-row core-matrix groups
  static constexpr int A_TILE = kRows * KP * 2;
  static constexpr int B_TILE = kEntries * KP * 2;
  static constexpr int RAW = TC * kTileTokens * kSpan * 2;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_A = OFF_B + NGC * B_TILE;
  static constexpr int OFF_RAW = OFF_A + 2 * NGC * A_TILE;   // A slots: [tile parity][group]
  static constexpr int OFF_NMAX = OFF_RAW + kRawStages * RAW;
  static constexpr int OFF_BAR = OFF_NMAX + 16 * 4;
  static constexpr int OFF_BMIN = OFF_BAR + 8 * (kRawStages + 2);     // [2 sets][8 blocks][128 rows]
  static constexpr int OFF_MASK = OFF_BMIN + 2 * (kEntries / 32) * kRows * 4;   // [2 sets][8 blocks][128 rows]
  static constexpr int OFF_TMEM = OFF_MASK + 2 * (kEntries / 32) * kRows * 4;
  // + alignment slack; at least 120 KB so that one CTA (holding all of TMEM) fits per SM
  static constexpr int SMEM = (OFF_TMEM + 16 + 1024) > 120 * 1024 ? (OFF_TMEM + 16 + 1024) : 120 * 1024;
  static_assert(NGC == 2 || NGC == 4, "two MMA sets alternate over the item's groups");
  static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");
  static_assert(KP % 16 == 0, "K steps");
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
__device__ inline void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(n) : "memory"); }

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

template <int G, int C>
__global__ void __launch_bounds__(kThreads, 1) encode_tc_kernel(
    const __grid_constant__ CUtensorMap tmap, Geo g, int layer, int req, int tok_begin, int n_tok,
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);  // [0..1] raw stages, [2..3] MMA sets
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + X::OFF_TMEM);
  volatile int* fail_s = reinterpret_cast<volatile int*>(smem + X::OFF_TMEM + 4);   // per MMA set
  float* bmin_s = reinterpret_cast<float*>(smem + X::OFF_BMIN);
  uint32_t* mask_s = reinterpret_cast<uint32_t*>(smem + X::OFF_MASK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int set = tid / kSetThreads;      // MMA set: warps 0-7 or 8-15
  const int hf = (warp >> 2) & 1;         // half of the 256 entries this warp scans
  const int row = 32 * (warp & 3) + lane; // TMEM lane = tile row = token of the tile
  const bool set_leader = (tid % kSetThreads) == 0;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" :: "r"(smem_addr(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kRawStages + 2; ++i) mbar_init(smem_addr(&bars[i]), 1);
    fence_mbar_init();
    fail_s[0] = 0;
    fail_s[1] = 0;
  }
  // zero the A tiles once: the columns past G + 3 stay zero
  for (int i = tid; i < 2 * NGC * X::A_TILE / 16; i += kThreads)
    reinterpret_cast<uint4*>(At)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_set = tmem_base + (uint32_t)(set * 256);
  const uint32_t lane_addr = ((uint32_t)(32 * (warp & 3))) << 16;
  float* const bmin_set = bmin_s + set * (kEntries / 32) * kRows;     // [8 blocks][128 rows]
  uint32_t* const mask_set = mask_s + set * (kEntries / 32) * kRows;  // [8 blocks][128 rows]

  const int n_spans = g.d / kSpan;
  const int n_sets = 2 * g.nblk * g.H * n_spans;
  const int n_ranges = (n_tok + kItemTokens - 1) / kItemTokens;
  const long n_items = (long)n_sets * n_ranges;

  // A row of this thread's token for group gib from a raw tile: element s*c+e =
  // raw[s][row][gib*c+e].  Both threads of a row read it (for ||x||^2); each writes half of
  // its 16-byte chunks.  Returns ||x||^2 of the joint vector.
  auto build_a = [&](const unsigned char* src_tile, int gib, unsigned char* at) -> float {
    uint32_t xw[G / 2];                  // the row's G elements, two per word
#pragma unroll
    for (int s2 = 0; s2 < TC; ++s2) {
      const unsigned char* src = src_tile + raw_off(s2, row, gib * C);
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
    float x2 = 0.f;
#pragma unroll
    for (int q = 0; q < G / 2; ++q) {
      const float lo = bf16_lo(xw[q]), hi = bf16_hi(xw[q]);
      x2 = fmaf(lo, lo, x2);
      x2 = fmaf(hi, hi, x2);
    }
#pragma unroll
    for (int k8 = 0; k8 < G / 8; ++k8)
      if ((k8 >= G / 16) == (hf == 1))
        *reinterpret_cast<uint4*>(at + kmaj_off(row, k8 * 8, SBO)) =
            make_uint4(xw[k8 * 4], xw[k8 * 4 + 1], xw[k8 * 4 + 2], xw[k8 * 4 + 3]);
    if (hf == 1) {
      const uint32_t one = 0x3f80u;   // bf16 1.0
      *reinterpret_cast<uint4*>(at + kmaj_off(row, G, SBO)) = make_uint4(one | (one << 16), one, 0u, 0u);
    }
    fence_proxy_async();             // the tile is read by the tensor core (async proxy)
    return x2;
  };
  // the set's UMMA of group gib from A slot aslot into the set's TMEM columns (one thread)
  auto issue_mma = [&](int aslot, int gib) {
    const uint32_t a0 = smem_addr(At + aslot * X::A_TILE), b0 = smem_addr(Bt + gib * X::B_TILE);
#pragma unroll
    for (int ks = 0; ks < X::KSTEPS; ++ks)
      mma_bf16(tmem_set, smem_desc(a0 + ks * 256, SBO), smem_desc(b0 + ks * 256, SBO), kIdesc, ks > 0);
    mma_commit(smem_addr(&bars[kRawStages + set]));
  };
  bool issued = false;              // the set's next MMA was issued during the previous group
  bool outstanding = false;         // an MMA of this set may still be running
  float xx_next = 0.f;

  uint32_t raw_phase = 0;   // bit s: parity of raw stage s
  uint32_t mma_phase = 0;
  int tile_counter = 0;     // tiles processed by this CTA (drives the raw ring)
  bool failed = false;

  for (long item = blockIdx.x; item < n_items && !failed; item += gridDim.x) {
    int cs = (int)(item / n_ranges);
    const int range = (int)(item % n_ranges);
    const int span = cs % n_spans; cs /= n_spans;
    const int h = cs % g.H; cs /= g.H;
    const int blk = cs % g.nblk; cs /= g.nblk;
    const int kvi = cs;
    const int t_first = tok_begin + range * kItemTokens;
    const int t_last = min(tok_begin + n_tok, t_first + kItemTokens);
    const int n_tiles = (t_last - t_first + kTileTokens - 1) / kTileTokens;
    uint8_t* const idx_item = idx + idx_stream_off(g, layer, blk, req, h, kvi);

    // all MMAs of the previous item have completed (each set waited for its commits)
    __syncthreads();
    // prefetch the first two raw tiles of this item
    if (tid == 0) {
      for (int tl = 0; tl < min(2, n_tiles); ++tl) {
        const int stg = (tile_counter + tl) % kRawStages;
        const uint32_t bar = smem_addr(&bars[stg]);
        mbar_expect_tx(bar, X::RAW);
        tma_load_3d(smem_addr(raw + stg * X::RAW), &tmap, h * g.d + span * kSpan, t_first + tl * kTileTokens,
                    kvi * g.T + blk * TC, bar);
      }
    }
    // B tiles: [-2 C_k | n1 n2 n3 | 0] for the item's groups, K-major no-swizzle;
    // nmax_s[gi] = max_k ||C_k||^2 (non-negative floats order like their bits)
    if (tid < NGC) nmax_s[tid] = 0.f;
    __syncthreads();
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

    for (int tl = 0; tl < n_tiles && !failed; ++tl, ++tile_counter) {
      const int stg = tile_counter % kRawStages;
      const int t0 = t_first + tl * kTileTokens;
      if (__syncthreads_or(!mbar_wait(smem_addr(&bars[stg]), (raw_phase >> stg) & 1u, g.wait_iters))) {
        failed = true;
        break;
      }
      raw_phase ^= 1u << stg;
      const unsigned char* rw = raw + stg * X::RAW;
      const bool valid_row = t0 + row < t_last;

      // each set handles groups gi = set, set + 2, ...  The A tile of the set's next group is
      // built while the current group's MMA runs (A slots alternate with the tile parity), and
      // that next MMA is issued as soon as the current one's accumulator has been read.
      for (int gi = set; gi < NGC; gi += 2) {
        const int slot = gi + NGC * (tile_counter & 1);
        float xx;
        if (issued) {
          xx = xx_next;
          issued = false;
        } else {
          xx = build_a(rw, gi, At + slot * X::A_TILE);
          tc_fence_before();
          named_sync(1 + set, kSetThreads);
          if (set_leader) issue_mma(slot, gi);
          outstanding = true;
        }
        int next_slot = -1, next_gi = 0;
        if (gi + 2 < NGC) {
          next_slot = slot + 2;
          next_gi = gi + 2;
          xx_next = build_a(rw, next_gi, At + next_slot * X::A_TILE);
        } else if (tl + 1 < n_tiles) {
          // the set's first group of the next tile: its raw stage was requested two tiles ago
          const int stg1 = (tile_counter + 1) % kRawStages;
          if (mbar_wait(smem_addr(&bars[stg1]), (raw_phase >> stg1) & 1u, g.wait_iters)) {
            next_slot = set + NGC * ((tile_counter + 1) & 1);
            next_gi = set;
            xx_next = build_a(raw + stg1 * X::RAW, set, At + next_slot * X::A_TILE);
          } else {
            fail_s[set] = 1;
          }
        }
        // one warp of the set waits for the MMA; the barrier releases the others (no spinning)
        if ((tid % kSetThreads) < 32) {
          __syncwarp();
          if (!mbar_wait(smem_addr(&bars[kRawStages + set]), mma_phase, g.wait_iters)) fail_s[set] = 1;
        }
        named_sync(1 + set, kSetThreads);
        tc_fence_after();

        // epilogue, one pass over this warp's half of the row (four 32-column blocks, two
        // 64-column loads): each block's minimum, and the block's columns within eps of that
        // minimum as a bit mask (bit 31 - i for column i).  Of the block holding the row
        // minimum, that mask is exactly the row's candidates inside it; of any other block it
        // holds every candidate of the row in that block (its minimum is not below the row's).
        const float eps = (xx + nmax_s[gi]) * 0x1p-14f;
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t ra[64];
          tmem_ld64_nowait(tmem_set + lane_addr + hf * 128 + q2 * 64, ra);
          tmem_wait_ld();
#pragma unroll
          for (int b2 = 0; b2 < 2; ++b2) {
            const uint32_t* r = ra + 32 * b2;
            float m0 = __uint_as_float(r[0]), m1 = __uint_as_float(r[1]);
#pragma unroll
            for (int i = 2; i < 30; i += 4) {          // columns 2..29
              m0 = fmin3(m0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
              m1 = fmin3(m1, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
            }
            m0 = fmin3(m0, __uint_as_float(r[30]), __uint_as_float(r[31]));
            const float bm = fminf(m0, m1);
            // sign of (bm + eps) - v per column, shifted in: 1 = outside the window
            const float tb = bm + eps;
            const float2 t2 = make_float2(tb, tb), neg1 = make_float2(-1.f, -1.f);
            uint32_t sg = 0u;
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 e = __ffma2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), neg1, t2);
              sg = __funnelshift_l(__float_as_uint(e.x), sg, 1);
              sg = __funnelshift_l(__float_as_uint(e.y), sg, 1);
            }
            const int q = hf * 4 + q2 * 2 + b2;
            bmin_set[q * kRows + row] = bm;
            mask_set[q * kRows + row] = ~sg;
          }
        }
        tc_fence_before();
        named_sync(1 + set, kSetThreads);      // also: every thread saw the MMA wait's outcome
        const bool ok = fail_s[set] == 0;      // uniform over the set
        if (ok) outstanding = false;
        mma_phase ^= 1u;                       // one completed phase of this set's barrier per group
        // the accumulator has been read: start the next group's MMA (its A tile was completed by
        // every thread of the set before the barrier above)
        if (ok && next_slot >= 0) {
          if (set_leader) {
            tc_fence_after();
            issue_mma(next_slot, next_gi);
          }
          issued = true;
          outstanding = true;
        }
        float bmin[kEntries / 32];
#pragma unroll
        for (int q = 0; q < kEntries / 32; ++q) bmin[q] = bmin_set[q * kRows + row];
        float mrow = bmin[0];
#pragma unroll
        for (int q = 1; q < kEntries / 32; ++q) mrow = fminf(mrow, bmin[q]);
        const float thr = mrow + eps;
        uint32_t bmask = 0, at_min = 0;   // blocks that can hold a candidate / that hold the minimum
#pragma unroll
        for (int q = 0; q < kEntries / 32; ++q) {
          bmask |= (bmin[q] <= thr ? 1u : 0u) << q;
          at_min |= (bmin[q] == mrow ? 1u : 0u) << q;
        }
        const int wb = at_min ? __ffs(at_min) - 1 : 0;   // the first block holding the minimum
        const bool mine = (wb >> 2) == hf;     // this thread's half holds it: it owns the row
        const uint32_t cm = mask_set[wb * kRows + row];
        int code = wb * 32 + __clz(cm);
        const bool tie = mine && valid_row && (__popc(cm) + __popc(bmask & ~(1u << wb)) > 1);
        if (tie) {
          // near-tie: exact fp64 direct-form distances of the candidates of every block within
          // eps (the block masks are supersets of them), lowest index on ties
          const unsigned char* bt = Bt + gi * X::B_TILE;
          double best = 1e300;
          int bk = kEntries;
          for (uint32_t wm = bmask; wm; wm &= wm - 1u) {
            const int q = __ffs(wm) - 1;
            for (uint32_t m = mask_set[q * kRows + row]; m; m &= m - 1u) {
              const int k = q * 32 + 32 - __ffs(m);       // bit 31 - i holds column i
              double d2 = 0.0;                           // sum_j (x_j - C_kj)^2; the tile holds -2 C
#pragma unroll
              for (int s2 = 0; s2 < TC; ++s2)
#pragma unroll
                for (int e = 0; e < C; ++e) {
                  const int j = s2 * C + e;
                  const uint32_t cw = *reinterpret_cast<const uint32_t*>(bt + kmaj_off(k, j & ~1, SBO));
                  const float c2 = (j & 1) ? bf16_hi(cw) : bf16_lo(cw);
                  const float xf = __bfloat162float(
                      *reinterpret_cast<const __nv_bfloat16*>(rw + raw_off(s2, row, gi * C + e)));
                  const double df = (double)xf + 0.5 * (double)c2;
                  d2 = fma(df, df, d2);
                }
              if (d2 < best || (d2 == best && k < bk)) { best = d2; bk = k; }
            }
          }
          code = bk;
        }
        if (mine && valid_row && ok) {
          const int cn = coded_offset + (t0 + row - tok_begin);
          idx_item[(size_t)(cn >> 3) * g.page_bytes + (span * NGC + gi) * kPage + (cn & 7)] = (uint8_t)code;
        }
        if (!ok) break;
      }
      fence_proxy_async();   // this thread's reads of the raw stage before its refill by TMA
      if (__syncthreads_or(fail_s[0] | fail_s[1])) failed = true;
      // refill this raw stage with the tile two ahead
      if (tid == 0 && tl + 2 < n_tiles) {
        const uint32_t bar = smem_addr(&bars[stg]);
        mbar_expect_tx(bar, X::RAW);
        tma_load_3d(smem_addr(raw + stg * X::RAW), &tmap, h * g.d + span * kSpan, t0 + 2 * kTileTokens,
                    kvi * g.T + blk * TC, bar);
      }
    }
  }
  if (failed && tid == 0) set_status(st, LVQ_ETIMEOUT);
  if (failed && set_leader && outstanding)   // let a set's last MMA finish before TMEM is freed
    mbar_wait(smem_addr(&bars[kRawStages + set]), mma_phase, g.wait_iters);
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
  CUtensorMap map;
  // dims: channels of a token row (H*d), tokens, (kv, step) planes
  cuuint64_t dims[3] = {(cuuint64_t)g.H * g.d, (cuuint64_t)kv_tokens, (cuuint64_t)2 * g.T};
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
  const long items = n_sets * ((n_tok + tc::kItemTokens - 1) / tc::kItemTokens);
  const int grid = (int)std::min<long>(items, n_sm[dev]);
  tc::encode_tc_kernel<G, C><<<grid, tc::kThreads, X::SMEM, s>>>(map, g, layer, req, tok_begin, n_tok,
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
