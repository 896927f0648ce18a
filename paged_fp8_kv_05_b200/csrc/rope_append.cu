// Fused rotary embedding + FP8 quantise + paged append, from the bf16 QKV
// projection output of the new tokens.
//
// The deep-dive page (Atlas: Rust/CUDA LLM inference engine, ainews.cool,
// "Kernel fusion" paragraph) fuses the steps of a transformer block into one
// kernel; this is the step in front of paged decode.  For every new token t of
// sequence b (position pos = start_pos[b] + t) and every head of its
// projection row [Hq query | Hkv key | Hkv value heads] x D (bf16):
//   * query and key heads are rotated ("rotate half": element i < D/2 pairs
//     with i + D/2; with c = cos_sin[pos][i], s = cos_sin[pos][D/2 + i]
//         out[i] = x[i] c - x[i + D/2] s,   out[i + D/2] = x[i + D/2] c + x[i] s
//     in float32, every product and sum rounded separately -- no fused
//     multiply-add -- so the value that decides an FP8 code is one exact
//     float32 number);
//   * the rotated query is written as bf16 (round to nearest even);
//   * the rotated key and the value are quantised to E4M3 with the per-KV-head
//     scale (IEEE division, round to nearest even, saturating) and scattered
//     into their pages exactly as atlas_fp8_kv_append does.
// HBM-bound: each projection row is read once (2 bytes per element), the
// cos/sin row of a position is shared by all heads of the token (L2), and
// each element leaves as 2 (query) or 1 (key, value) bytes.
#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kThreads = 256;

template <int D>
__global__ void __launch_bounds__(kThreads) rope_append_kernel(const RopeAppendParams p) {
  constexpr int TPR = D / 16;          // threads per head row: 8 pairs of columns each
  constexpr int H2 = D / 2;
  const int heads = p.Hq + 2 * p.Hkv;
  const long long row = (long long)blockIdx.x * (kThreads / TPR) + threadIdx.x / TPR;
  const int c = threadIdx.x % TPR;     // columns [8c, 8c + 8) and [D/2 + 8c, D/2 + 8c + 8)
  const long long rows = (long long)p.batch * p.n_new * heads;
  if (row >= rows) return;
  const int head = (int)(row % heads);
  const long long bt = row / heads;    // b * n_new + t
  const int t = (int)(bt % p.n_new), b = (int)(bt / p.n_new);
  const int pos = __ldg(p.start_pos + b) + t;
  const bool is_v = head >= p.Hq + p.Hkv;

  // the projection row: 8 bf16 from each half, as exact float32
  const __nv_bfloat16* src = p.qkv + (size_t)row * D;
  float x[16];
  {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(src + 8 * c));
    const uint4 z = __ldg(reinterpret_cast<const uint4*>(src + H2 + 8 * c));
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(wa[k] << 16);
      x[2 * k + 1] = __uint_as_float(wa[k] & 0xFFFF0000u);
      x[8 + 2 * k] = __uint_as_float(wz[k] << 16);
      x[8 + 2 * k + 1] = __uint_as_float(wz[k] & 0xFFFF0000u);
    }
  }
  if (pos < 0 || pos >= p.max_pos) {  // the whole token is skipped
    if (c == 0) atomicOr(p.err, ATLAS_DEVERR_APPEND);
    return;
  }
  if (!is_v) {
    const float* cs = p.cos_sin + (size_t)pos * D;
    const float4 c0 = __ldg(reinterpret_cast<const float4*>(cs + 8 * c));
    const float4 c1 = __ldg(reinterpret_cast<const float4*>(cs + 8 * c + 4));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(cs + H2 + 8 * c));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(cs + H2 + 8 * c + 4));
    const float co[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float si[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float x1 = x[k], x2 = x[8 + k];
      x[k] = __fsub_rn(__fmul_rn(x1, co[k]), __fmul_rn(x2, si[k]));
      x[8 + k] = __fadd_rn(__fmul_rn(x2, co[k]), __fmul_rn(x1, si[k]));
    }
  }
  if (head < p.Hq) {  // rotated query -> bf16
    __nv_bfloat16* dst = p.q_out + ((size_t)bt * p.Hq + head) * D;
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __nv_bfloat162 v2 = __floats2bfloat162_rn(x[2 * k], x[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t*>(&v2);
    }
    *reinterpret_cast<uint4*>(dst + 8 * c) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(dst + H2 + 8 * c) = make_uint4(w[4], w[5], w[6], w[7]);
    return;
  }
  // key or value: quantise and scatter (positions outside the table row or
  // with a bad page id are skipped and flagged)
  const int h = is_v ? head - p.Hq - p.Hkv : head - p.Hq;
  const int blk = pos / p.ps;
  int page = -1;
  if (pos >= 0 && blk < p.max_blocks) page = __ldg(p.block_table + (size_t)b * p.max_blocks + blk);
  if (page < 0 || page >= p.num_pages) {
    if (c == 0) atomicOr(p.err, ATLAS_DEVERR_APPEND);
    return;
  }
  const uint4 codes = quantize16_e4m3(x, __ldg((is_v ? p.v_scale : p.k_scale) + h));
  const size_t head_page = (size_t)page * p.Hkv + h;
  const int slot = pos % p.ps;
  if (!is_v) {
    // dims [8c, 8c + 8) and [D/2 + 8c, ...): half of 16-byte chunk 8c / 16 and
    // of chunk (D/2 + 8c) / 16, placed by the K page layout
    uint8_t* rowp = p.k_pages + (head_page * p.ps + slot) * D;
    const int j0 = (8 * c) / 16, j1 = (H2 + 8 * c) / 16, sub = (8 * c) % 16;
    *reinterpret_cast<uint2*>(rowp + 16 * k_chunk_pos(D, slot, j0) + sub) =
        make_uint2(codes.x, codes.y);
    *reinterpret_cast<uint2*>(rowp + 16 * k_chunk_pos(D, slot, j1) + sub) =
        make_uint2(codes.z, codes.w);
  } else {
    // V pages: 16-slot groups, head-dim-major: byte group_pos(slot % 16) of the
    // group row of each head dimension
    const int t16 = slot % 16;
    const int byte = 4 * ((t16 & 7) >> 1) + 2 * (t16 >> 3) + (t16 & 1);
    uint8_t* grp = p.v_pages + (head_page * (p.ps / 16) + slot / 16) * (16 * D) + byte;
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int d = (k < 8) ? 8 * c + k : H2 + 8 * c + (k - 8);
      grp[16 * d] = (uint8_t)(w[k >> 2] >> (8 * (k & 3)));
    }
  }
}

}  // namespace

cudaError_t launch_rope_append(const RopeAppendParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.batch * p.n_new * (p.Hq + 2 * p.Hkv);
  if (rows <= 0) return cudaSuccess;
  const int rows_per_cta = kThreads / (p.D / 16);
  const long long grid = (rows + rows_per_cta - 1) / rows_per_cta;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (p.D == 128)
    rope_append_kernel<128><<<(unsigned)grid, kThreads, 0, stream>>>(p);
  else if (p.D == 64)
    rope_append_kernel<64><<<(unsigned)grid, kThreads, 0, stream>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace atlas
