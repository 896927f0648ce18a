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

__device__ __forceinline__ void load16_as_f32(const void* base, size_t elem, int dtype,
                                              float (&x)[16]) {
  if (dtype == ATLAS_DTYPE_F32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 v = __ldg(p + i);
      x[4 * i + 0] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(
        static_cast<const __nv_bfloat16*>(base) + elem);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint4 v = __ldg(p + i);
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {   // bf16 -> f32 is exact: the bits move up 16
        x[8 * i + 2 * k + 0] = __uint_as_float(w[k] << 16);
        x[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  }
}

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
    const float sc = __ldg((which ? p.v_scale : p.k_scale) + h);

    uint32_t packed[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float y0 = __fdiv_rn(x[4 * w + 0], sc);
      const float y1 = __fdiv_rn(x[4 * w + 1], sc);
      const float y2 = __fdiv_rn(x[4 * w + 2], sc);
      const float y3 = __fdiv_rn(x[4 * w + 3], sc);
      const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(y2, y3), __NV_SATFINITE, __NV_E4M3);
      packed[w] = (lo & 0xFFFFu) | (hi << 16);
    }
    if (!which) {
      uint8_t* dst = p.k_pages + (((size_t)page * p.Hkv + h) * p.ps + (pos % p.ps)) * p.D + 16 * j;
      *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    } else {
      const int slot = pos % p.ps, t = slot % 16;
      const int byte = 4 * ((t & 7) >> 1) + 2 * (t >> 3) + (t & 1);
      uint8_t* dst = p.v_pages + (((size_t)page * p.Hkv + h) * (p.ps / 16) + slot / 16) * (16 * p.D) +
                     (size_t)(16 * j) * 16 + byte;
#pragma unroll
      for (int k = 0; k < 16; ++k) dst[16 * k] = (uint8_t)(packed[k >> 2] >> (8 * (k & 3)));
    }
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
