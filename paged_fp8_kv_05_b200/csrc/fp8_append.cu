// FP8 page append: quantise new K/V rows to E4M3 with a per-KV-head scale and
// scatter them into their pages through the block table.
//
// Source: the FP8 KV quantisation with scale factors of the Atlas deep-dive
// (ainews.cool, "Quantisation" paragraph) and the paged FP8 KV cache of the
// GB10 page (ainews.surl.tw).  Encoding reading: y = fp32(x) / fp32(scale[h])
// as an IEEE round-to-nearest division (__fdiv_rn, never a reciprocal
// multiply), then round-to-nearest-even to E4M3 with saturation to +-448
// (cvt.rn.satfinite), sign of zero kept.  The result must be bit-exact with
// that definition.
//
// Page layouts: K pages are token-major [P][Hkv][ps][D]; V pages are kept in
// groups of 16 slots, head-dim-major inside a group: [P][Hkv][ps/16][D][16]
// (16 consecutive tokens of one head dimension adjacent), slot t of a group at
// byte 4*((t%8)/2) + 2*(t/8) + t%2 (bytes 4c..4c+3 hold slots 2c, 2c+1, 2c+8,
// 2c+9, the token order of the decode kernel's P fragments).
// Memory-bound: per element 4 (f32) or 2 (bf16) bytes read, 1 byte written.
// One thread owns 16 consecutive elements of one (sequence, token, head) row:
// 64 B (or 32 B) of coalesced input, then one 16-byte store into a K page or
// 16 byte stores (one per head dimension, 16 bytes apart) into a V page.
#include "atlas_internal.cuh"

namespace atlas {
namespace {

__global__ void __launch_bounds__(256) fp8_append_kernel(const AppendParams p) {
  const int chunks = p.D / 16;
  const long long per_tensor = (long long)p.batch * p.n_new * p.Hkv * chunks;
  const long long total = 2 * per_tensor;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += stride) {
    const int which = idx >= per_tensor;   // 0 = K, 1 = V
    long long r = idx - (which ? per_tensor : 0);
    const int j = (int)(r % chunks); r /= chunks;
    const int h = (int)(r % p.Hkv); r /= p.Hkv;
    const int t = (int)(r % p.n_new);
    const int b = (int)(r / p.n_new);

    const int pos = __ldg(p.start_pos + b) + t;
    const int blk = pos / p.ps;
    if (pos < 0 || blk >= p.max_blocks) { atomicOr(p.err, ATLAS_DEVERR_APPEND); continue; }
    const int page = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
    if (page < 0 || page >= p.num_pages) { atomicOr(p.err, ATLAS_DEVERR_APPEND); continue; }

    const size_t src_elem = ((((size_t)b * p.n_new + t) * p.Hkv + h) * p.D) + 16 * j;
    float x[16];
    load16_as_f32(which ? p.v_new : p.k_new, src_elem, p.dtype, x);
    const uint4 codes = quantize16_e4m3(x, __ldg((which ? p.v_scale : p.k_scale) + h));
    const size_t head_page = (size_t)page * p.Hkv + h;
    if (!which)
      store16_k(p.k_pages, head_page, p.D, p.ps, pos % p.ps, j, codes);
    else
      store16_v(p.v_pages, head_page, p.D, p.ps, pos % p.ps, j, codes);
  }
}

}  // namespace

cudaError_t launch_fp8_append(const AppendParams& p, int num_sms, cudaStream_t stream) {
  const long long total = 2LL * p.batch * p.n_new * p.Hkv * (p.D / 16);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  long long blocks = (total + threads - 1) / threads;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  fp8_append_kernel<<<(unsigned)blocks, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace atlas
