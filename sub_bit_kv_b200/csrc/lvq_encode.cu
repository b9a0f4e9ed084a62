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
    uint8_t* __restrict__ idx, int32_t* st) {
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
  const int phys = phys_page(g, req, cn >> 3);
  if (phys < 0) {
    set_status(st, LVQ_ECAPACITY);
    return;
  }
  idx[idx_code_off(g, layer, blk, req, h, kvi, phys, cn, grp)] = (uint8_t)bk;
}

template <int G, int C>
static cudaError_t encode_prefill_as(const Geo& g, int layer, int req, const __nv_bfloat16* kv,
                                     int64_t tok_stride, int kv_tokens, int tok_begin, int n_tok,
                                     int coded_offset, const __nv_bfloat16* cb, uint8_t* idx,
                                     int32_t* st, cudaStream_t s) {
  dim3 grid((n_tok + kEncThreads - 1) / kEncThreads, 2 * g.nblk * g.H * g.ng);
  encode_prefill_kernel<G, C><<<grid, kEncThreads, 0, s>>>(g, layer, req, kv, tok_stride, kv_tokens,
                                                            tok_begin, n_tok, coded_offset, cb, idx, st);
  return cudaGetLastError();
}

bool encode_supported(int G, int c) {
  return (G == 16 || G == 32) && (c == 4 || c == 8 || c == 16) && c <= G;
}

cudaError_t launch_encode_prefill(const Geo& g, int layer, int req, const __nv_bfloat16* kv,
                                  int64_t tok_stride, int kv_tokens, int tok_begin, int n_tok,
                                  int coded_offset, const __nv_bfloat16* cb, uint8_t* idx,
                                  int32_t* st, cudaStream_t s) {
  if (n_tok == 0) return cudaSuccess;
  if (layer < 0) {   // every layer: kv holds the layers back to back, one launch each
    const int64_t layer_stride = (int64_t)2 * g.T * kv_tokens * tok_stride;
    for (int l = 0; l < g.L; ++l) {
      const cudaError_t e = launch_encode_prefill(g, l, req, kv + l * layer_stride, tok_stride, kv_tokens, tok_begin,
                                                  n_tok, coded_offset, cb, idx, st, s);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
#define LVQ_ENC(GG, CC)                                                                          \
  if (g.G == GG && g.c == CC)                                                                    \
    return encode_prefill_as<GG, CC>(g, layer, req, kv, tok_stride, kv_tokens, tok_begin, n_tok, \
                                     coded_offset, cb, idx, st, s);
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

// Page encode.  A codebook's contraction with one page is small -- 8 vectors
// (the page's tokens) x 256 entries x G -- and every page encode touches every
// codebook of every layer (201 MB of bf16 at the Ouro-1.4B shapes), so the
// kernel is built to stream codebooks: a persistent grid whose warps each walk
// a strided list of codebooks, every codebook (and its fp32 norms) bulk-copied
// into a 3-deep ring private to the warp, and one tensor-core MMA
// (mma.sync m16n8k16, bf16 in, fp32 accumulate) per 16 entries x 8 vectors x
// 16 dimensions, with the page's 8 tokens as the N = 8 columns.  For every
// request whose page is due the warp then takes the fp32 expansion form
// n_k - 2 x.C_k; every entry within eps = 2^-14 (||x||^2 + max_k n_k) of the
// minimum is a candidate (the fp32 error is far below eps), and when there are
// several they are rescored exactly in the fp64 direct form, lowest index on
// ties.
template <int G, int C>
struct PageEnc {
  static constexpr int TC = G / C;
  static constexpr int NW = G == 16 ? 8 : 4;          // warps per CTA
  static constexpr int NBUF = 3;                      // codebooks in flight per warp
  static constexpr int CBB = kEntries * G * 2;        // one codebook, bf16
  static constexpr int NB = kEntries * 4;             // its fp32 squared norms
  static constexpr int BUF = CBB + NB;
  static constexpr int KS = G / 16;                   // MMA k-steps
  static constexpr int MAXB = kPageMaxBatch;
  static constexpr int OFF_BAR = NW * NBUF * BUF;
  static constexpr int OFF_DUE = OFF_BAR + NW * NBUF * 8;
  static constexpr int SMEM = OFF_DUE + 2 * MAXB * 4 + 16;
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(BUF % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
};

__device__ inline void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ inline void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

template <int G, int C>
__global__ void __launch_bounds__(PageEnc<G, C>::NW * 32, 1) encode_page_kernel(
    Geo g, int batch, const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ coded_len,
    const __nv_bfloat16* __restrict__ ring, const __nv_bfloat16* __restrict__ cb,
    const float* __restrict__ cb_norm, uint8_t* __restrict__ idx, int32_t* st) {
  using X = PageEnc<G, C>;
  constexpr int TC = X::TC, NW = X::NW, NBUF = X::NBUF, KS = X::KS;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + X::OFF_BAR);
  int* due = reinterpret_cast<int*>(smem + X::OFF_DUE);     // [n_due] requests, then [n_due] coded_len
  int* n_due_s = due + 2 * X::MAXB;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    int n = 0;
    for (int b = 0; b < batch; ++b) {
      const int d = page_due(g, ctx_len[b], coded_len[b]);
      if (d < 0 && blockIdx.x == 0) set_status(st, LVQ_ECAPACITY);
      if (d == 1) {
        due[n] = b;
        due[X::MAXB + n] = coded_len[b];
        ++n;
      }
    }
    *n_due_s = n;
    for (int i = 0; i < NW * NBUF; ++i) mbar_init(smem_addr(&bars[i]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int n_due = *n_due_s;
  if (n_due == 0) return;

  const long n_cb = (long)g.L * 2 * g.nblk * g.H * g.ng;   // codebooks, (layer, kv, blk, h, grp) order
  const long stride = (long)gridDim.x * NW;
  const long first = (long)blockIdx.x * NW + warp;
  unsigned char* wbuf = smem + (size_t)warp * NBUF * X::BUF;
  uint64_t* wbar = bars + warp * NBUF;

  auto issue = [&](long c, int slot) {            // lane 0: codebook c into ring slot `slot`
    const uint32_t bar = smem_addr(&wbar[slot]);
    mbar_expect_tx(bar, X::BUF);
    bulk_g2s(smem_addr(wbuf + slot * X::BUF), cb + (size_t)c * kEntries * G, X::CBB, bar);
    bulk_g2s(smem_addr(wbuf + slot * X::BUF + X::CBB), cb_norm + (size_t)c * kEntries, X::NB, bar);
  };
  if (lane == 0)
    for (int i = 0; i < NBUF - 1; ++i)
      if (first + i * stride < n_cb) issue(first + i * stride, i);

  const int q = lane & 3, r8 = lane >> 2;          // C fragment: vectors 2q, 2q+1; entries r8 (+8) of each 16
  for (long it = 0;; ++it) {
    const long c = first + it * stride;
    if (c >= n_cb) break;
    const int slot = (int)(it % NBUF);
    if (lane == 0 && c + (NBUF - 1) * stride < n_cb) issue(c + (NBUF - 1) * stride, (int)((it + NBUF - 1) % NBUF));
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_addr(&wbar[slot]), (uint32_t)((it / NBUF) & 1), g.wait_iters));
    if (!ok) {
      if (lane == 0) {
        set_status(st, LVQ_ETIMEOUT);
        for (long j = it; j < it + NBUF && first + j * stride < n_cb; ++j)   // copies still in flight
          mbar_wait(smem_addr(&wbar[j % NBUF]), (uint32_t)((j / NBUF) & 1), g.wait_iters);
      }
      break;
    }
    const unsigned char* cbs = wbuf + slot * X::BUF;
    const float* nrm = reinterpret_cast<const float*>(cbs + X::CBB);
    long cc = c;
    const int grp = (int)(cc % g.ng); cc /= g.ng;
    const int h = (int)(cc % g.H); cc /= g.H;
    const int blk = (int)(cc % g.nblk); cc /= g.nblk;
    const int kvi = (int)(cc % 2);
    const int layer = (int)(cc / 2);

    // squared norms this lane needs, and their maximum over the codebook
    float nr[16][2];
    float nmax = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      nr[m][0] = nrm[16 * m + r8];
      nr[m][1] = nrm[16 * m + r8 + 8];
      nmax = fmaxf(nmax, fmaxf(nr[m][0], nr[m][1]));
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) nmax = fmaxf(nmax, __shfl_xor_sync(0xffffffffu, nmax, o));

    for (int di = 0; di < n_due; ++di) {
      const int b = due[di], coded = due[X::MAXB + di];
      // B fragments: vector n = lane/4 (the page's token n), dimensions 16 ks + 2q (+1) and +8 (+9)
      const int slot_n = (coded + r8) % g.R;
      uint32_t bf[KS][2];
      float xxp = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int k = 16 * ks + 2 * q + 8 * hh;
          const int s2 = k / C, e = k % C;
          const __nv_bfloat16* p = ring + ring_off(g, layer, kvi, blk * TC + s2, b, h, slot_n) + grp * C + e;
          const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
          bf[ks][hh] = w;
          xxp = fmaf(bf16_lo(w), bf16_lo(w), xxp);
          xxp = fmaf(bf16_hi(w), bf16_hi(w), xxp);
        }
      xxp += __shfl_xor_sync(0xffffffffu, xxp, 1);
      xxp += __shfl_xor_sync(0xffffffffu, xxp, 2);          // ||x_n||^2 in the lanes of vector n
      const float xx0 = __shfl_sync(0xffffffffu, xxp, 4 * (2 * q));
      const float xx1 = __shfl_sync(0xffffffffu, xxp, 4 * (2 * q + 1));
      // d[m][0..3]: entries 16m + r8 (vectors 2q, 2q+1) and 16m + r8 + 8 (vectors 2q, 2q+1)
      float d[16][4];
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        d[m][0] = d[m][1] = d[m][2] = d[m][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a[4];
          const int mi = lane >> 3, rr = lane & 7;
          const int entry = 16 * m + (mi & 1) * 8 + rr, col = 16 * ks + (mi >> 1) * 8;
          ldmatrix_x4(a, smem_addr(cbs + entry * (2 * G) + col * 2));
          mma_bf16_16816(d[m], a, bf[ks][0], bf[ks][1]);
        }
        d[m][0] = fmaf(-2.f, d[m][0], nr[m][0]);
        d[m][1] = fmaf(-2.f, d[m][1], nr[m][0]);
        d[m][2] = fmaf(-2.f, d[m][2], nr[m][1]);
        d[m][3] = fmaf(-2.f, d[m][3], nr[m][1]);
      }
      float best0 = INFINITY, best1 = INFINITY;
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        best0 = fminf(best0, fminf(d[m][0], d[m][2]));
        best1 = fminf(best1, fminf(d[m][1], d[m][3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        best0 = fminf(best0, __shfl_xor_sync(0xffffffffu, best0, o));
        best1 = fminf(best1, __shfl_xor_sync(0xffffffffu, best1, o));
      }
      const float thr0 = best0 + (xx0 + nmax) * 6.103515625e-05f;   // 2^-14
      const float thr1 = best1 + (xx1 + nmax) * 6.103515625e-05f;
      // candidates as bit masks: bit 2m + hh is entry 16m + r8 + 8hh (increasing with the bit)
      uint32_t mk0 = 0u, mk1 = 0u;
#pragma unroll
      for (int m = 0; m < 16; ++m)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (d[m][2 * hh] <= thr0) mk0 |= 1u << (2 * m + hh);
          if (d[m][2 * hh + 1] <= thr1) mk1 |= 1u << (2 * m + hh);
        }
      auto entry_of = [&](int bit) { return 16 * (bit >> 1) + r8 + 8 * (bit & 1); };
      int n0 = __popc(mk0), n1 = __popc(mk1);
      int k0 = mk0 ? entry_of(__ffs(mk0) - 1) : kEntries;
      int k1 = mk1 ? entry_of(__ffs(mk1) - 1) : kEntries;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        n0 += __shfl_xor_sync(0xffffffffu, n0, o);
        n1 += __shfl_xor_sync(0xffffffffu, n1, o);
        k0 = min(k0, __shfl_xor_sync(0xffffffffu, k0, o));
        k1 = min(k1, __shfl_xor_sync(0xffffffffu, k1, o));
      }
      if (__any_sync(0xffffffffu, n0 > 1 || n1 > 1)) {
        // near-tie: exact fp64 direct-form distances of the candidates, lowest index on ties
#pragma unroll 1
        for (int v = 0; v < 2; ++v) {
          const bool tie = v == 0 ? n0 > 1 : n1 > 1;
          uint32_t mk = tie ? (v == 0 ? mk0 : mk1) : 0u;
          double bd = 1e300;
          int bk = kEntries;
          if (mk) {
            double x[G];
            const int slot_v = (coded + 2 * q + v) % g.R;
#pragma unroll
            for (int k = 0; k < G; ++k) {
              const int s2 = k / C, e = k % C;
              x[k] = (double)__bfloat162float(
                  ring[ring_off(g, layer, kvi, blk * TC + s2, b, h, slot_v) + grp * C + e]);
            }
            while (mk) {
              const int bit = __ffs(mk) - 1;
              mk &= mk - 1u;
              const int e = entry_of(bit);
              const __nv_bfloat16* ce = reinterpret_cast<const __nv_bfloat16*>(cbs) + e * G;
              double acc = 0.0;
#pragma unroll
              for (int k = 0; k < G; ++k) {
                const double df = x[k] - (double)__bfloat162float(ce[k]);
                acc = fma(df, df, acc);
              }
              if (acc < bd || (acc == bd && e < bk)) { bd = acc; bk = e; }
            }
          }
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            const double ob = __shfl_xor_sync(0xffffffffu, bd, o);
            const int ok2 = __shfl_xor_sync(0xffffffffu, bk, o);
            if (ob < bd || (ob == bd && ok2 < bk)) { bd = ob; bk = ok2; }
          }
          if (tie) {
            if (v == 0) k0 = bk;
            else k1 = bk;
          }
        }
      }
      if (r8 == 0) {                            // this lane's two tokens (coded_len need not be a multiple of 8)
        const int n = coded + 2 * q;
        // the 8 tokens may straddle two logical pages (coded_len need not be a multiple of 8)
        const int p0 = phys_page(g, b, n >> 3), p1 = phys_page(g, b, (n + 1) >> 3);
        if (p0 < 0 || p1 < 0) set_status(st, LVQ_ECAPACITY);
        if (p0 >= 0) idx[idx_code_off(g, layer, blk, b, h, kvi, p0, n, grp)] = (uint8_t)k0;
        if (p1 >= 0) idx[idx_code_off(g, layer, blk, b, h, kvi, p1, n + 1, grp)] = (uint8_t)k1;
      }
    }
    fence_proxy_async_shared();                 // this warp's reads of the slot precede its refill
    __syncwarp();
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
                                  const __nv_bfloat16* ring, const __nv_bfloat16* cb, const float* cb_norm,
                                  uint8_t* idx, int32_t* st, cudaStream_t s) {
  using X = PageEnc<G, C>;
  static int n_sm[kMaxDevices] = {};
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(encode_page_kernel<G, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, X::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  encode_page_kernel<G, C><<<n_sm[dev], X::NW * 32, X::SMEM, s>>>(g, batch, ctx_len, coded_len, ring, cb, cb_norm,
                                                                   idx, st);
  return cudaGetLastError();
}

cudaError_t launch_encode_page(const Geo& g, int batch, const int32_t* ctx_len, int32_t* coded_len,
                               const __nv_bfloat16* ring, const __nv_bfloat16* cb, const float* cb_norm,
                               uint8_t* idx, int32_t* st, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  cudaError_t e = cudaErrorInvalidValue;
#define LVQ_PG(GG, CC) \
  if (g.G == GG && g.c == CC) e = encode_page_as<GG, CC>(g, batch, ctx_len, coded_len, ring, cb, cb_norm, idx, st, s);
  LVQ_PG(16, 4) LVQ_PG(16, 8) LVQ_PG(16, 16) LVQ_PG(32, 4) LVQ_PG(32, 8) LVQ_PG(32, 16)
#undef LVQ_PG
  if (e != cudaSuccess) return e;
  advance_kernel<<<1, 256, 0, s>>>(g, batch, ctx_len, coded_len);
  return cudaGetLastError();
}

}  // namespace lvq
