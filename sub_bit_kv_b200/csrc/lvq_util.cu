// Layout helpers: codebook packing, RoPE tables, and the dequantisation test hook.
#include "lvq_common.cuh"

namespace lvq {

// cbp[layer][kv][blk][h][s][k][g][e] = cb[layer][kv][blk][h][g][k][s*c + e]
// ("LoopVQ summary", "premises and limits": attention at step t reads only the
// step-t slice of each entry, so each step's slice is made contiguous).
__global__ void pack_kernel(Geo g, const __nv_bfloat16* __restrict__ cb, __nv_bfloat16* __restrict__ cbp,
                            float* __restrict__ cb_norm) {
  const size_t n_sets = (size_t)g.L * 2 * g.nblk * g.H;     // (layer, kv, blk, h)
  const size_t per_set = (size_t)g.ng * kEntries * g.G;
  const size_t total = n_sets * per_set;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    size_t set = i / per_set, r = i % per_set;
    int j = (int)(r % g.G);
    int k = (int)((r / g.G) % kEntries);
    int grp = (int)(r / ((size_t)g.G * kEntries));
    int s = j / g.c, e = j % g.c;
    size_t dst = set * per_set + (((size_t)s * kEntries + k) * g.ng + grp) * g.c + e;
    cbp[dst] = cb[i];
  }
  if (!cb_norm) return;
  const size_t n_entries = n_sets * g.ng * kEntries;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n_entries; i += (size_t)gridDim.x * blockDim.x) {
    const __nv_bfloat16* e = cb + i * g.G;
    double acc = 0.0;
    for (int j = 0; j < g.G; ++j) {
      double v = (double)__bfloat162float(e[j]);
      acc += v * v;
    }
    cb_norm[i] = (float)acc;
  }
}

cudaError_t launch_pack(const Geo& g, const __nv_bfloat16* cb, __nv_bfloat16* cbp, float* cb_norm,
                        cudaStream_t s) {
  pack_kernel<<<1184, 256, 0, s>>>(g, cb, cbp, cb_norm);
  return cudaGetLastError();
}

// coarse[r][f] = (cos, sin)(8 r theta_f), fine[r][f] = (cos, sin)(r theta_f),
// theta_f = base^(-2f/d), evaluated in fp64 and rounded to fp32.
__global__ void rope_kernel(Geo g, double base, float* __restrict__ rope) {
  const int F = g.d / 2;
  const int rows = g.RC + kPage;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < rows * F; i += gridDim.x * blockDim.x) {
    int r = i / F, f = i % F;
    double theta = pow(base, -2.0 * (double)f / (double)g.d);
    double pos = (r < g.RC) ? 8.0 * (double)r : (double)(r - g.RC);
    double sn, cs;
    sincos(pos * theta, &sn, &cs);
    rope[2 * (size_t)i] = (float)cs;
    rope[2 * (size_t)i + 1] = (float)sn;
  }
}

cudaError_t launch_rope_table(const Geo& g, float base, float* rope, cudaStream_t s) {
  rope_kernel<<<592, 256, 0, s>>>(g, (double)base, rope);
  return cudaGetLastError();
}

// out[n][h][g*c + e] = step-t share of entry idx(n, h, g)
__global__ void dequant_kernel(Geo g, int layer, int step, int req, int kv, const uint8_t* __restrict__ idx,
                               const __nv_bfloat16* __restrict__ cbp, int tok_begin, int n_tok,
                               __nv_bfloat16* __restrict__ out) {
  const int blk = step / g.Tc, s = step % g.Tc;
  const size_t total = (size_t)n_tok * g.H * g.d;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    int ch = (int)(i % g.d);
    int h = (int)((i / g.d) % g.H);
    int n = tok_begin + (int)(i / ((size_t)g.d * g.H));
    int grp = ch / g.c, e = ch % g.c;
    const int phys = phys_page(g, req, n >> 3);
    const int code = phys < 0 ? 0 : idx[idx_code_off(g, layer, blk, req, h, kv, phys, n, grp)];
    const __nv_bfloat16* slice = cbp + cbp_slice_off(g, layer, kv, blk, h, s);
    out[i] = slice[((size_t)code * g.ng + grp) * g.c + e];
  }
}

cudaError_t launch_dequantize(const Geo& g, int layer, int step, int req, int kv, const uint8_t* idx,
                              const __nv_bfloat16* cbp, int tok_begin, int n_tok,
                              __nv_bfloat16* out, cudaStream_t s) {
  if (n_tok == 0) return cudaSuccess;
  dequant_kernel<<<592, 256, 0, s>>>(g, layer, step, req, kv, idx, cbp, tok_begin, n_tok, out);
  return cudaGetLastError();
}

}  // namespace lvq
