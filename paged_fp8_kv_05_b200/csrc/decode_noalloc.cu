// Decode / MTP-verify attention without any device allocation by the caller.
//
// Some callers cannot allocate device memory for a workspace: code that runs
// inside a host framework which owns every allocation (a plugin, an embedded
// runtime handed only input and output buffers), or a code path that must not
// touch the allocator at all.  For them, atlas_paged_gqa_decode_noalloc runs
// the same decode kernel as atlas_paged_gqa_decode but keeps its scratch --
// the split-KV partial results, the per-(sequence, KV head, row group)
// completion counters and the device error word -- in one file-scope
// __device__ array of kScratchBytes bytes.  Every GPU that loads the library
// holds that array until the process exits.  Nothing here calls cudaMalloc,
// cudaFree or any allocating routine.
//
// The array is shared by every call on a device and keeps the last call's
// contents; each call clears the counters and the error word (the only parts
// that must start at zero) with cudaMemsetAsync on its stream before the
// launch.  Calls whose kernels overlap on the GPU (different streams, no
// ordering) race on the array.  If the split-KV partials of the automatic
// partition would not fit, the call runs one CTA per (sequence, KV head, row
// group) segment, which writes no partials; a call that would then need a
// segment longer than 65536 tokens is rejected with ATLAS_ERR_WORKSPACE.
// The first call on a device looks up the array's device address
// (cudaGetSymbolAddress) with that device current; make that first call
// before any stream capture.  Device-side checks still zero the rows of an
// invalid sequence and skip bad page ids, but this variant has no error word
// the caller can read.
#include <math.h>

#include <mutex>

#include "atlas_internal.cuh"

namespace {

constexpr size_t kScratchBytes = 8u << 20;  // 8 MiB per GPU
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;
// Longest segment the one-CTA-per-segment fallback accepts.  Its CTA keeps a
// table of the segment's 32-token units in shared memory: 65536 tokens make
// 2048 entries of 8 bytes (16 KB), well inside the kernel's shared-memory
// budget.  (atlas::kMaxUnitsPerCta bounds the ranges of the balanced
// partition, which this fallback does not use.)
constexpr int kMaxWholeSegmentTokens = 65536;

__device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up once).
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

}  // namespace

extern "C" atlas_status_t atlas_paged_gqa_decode_noalloc(
    const void* q, const void* k_pages, const void* v_pages, const float* k_scale,
    const float* v_scale, const int32_t* block_table, int32_t max_blocks_per_seq,
    const int32_t* seq_lens, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t page_size, int32_t num_pages, int32_t q_len, int32_t max_seq_len,
    float sm_scale, void* out, void* stream) {
  if (batch < 0 || num_kv_heads < 1 || num_q_heads < 1 || num_q_heads % num_kv_heads != 0 ||
      q_len < 1 || num_pages < 1 || max_blocks_per_seq < 1 || max_seq_len < q_len)
    return ATLAS_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
  if (page_size < 16 || page_size > 1024 || page_size % 16 != 0) return ATLAS_ERR_UNSUPPORTED;
  if ((long long)max_seq_len > (long long)max_blocks_per_seq * page_size) return ATLAS_ERR_INVALID_ARG;
  if (!(sm_scale == sm_scale) || isinf(sm_scale)) return ATLAS_ERR_INVALID_ARG;
  if (batch == 0) return ATLAS_OK;
  if (!q || !k_pages || !v_pages || !k_scale || !v_scale || !block_table || !seq_lens || !out)
    return ATLAS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_pages) || !aligned16(v_pages))
    return ATLAS_ERR_INVALID_ARG;

  int sms = 148;
  {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      sms = n;
  }
  const int R = q_len * (num_q_heads / num_kv_heads);

  // the automatic partition of the pool-based entry point if its scratch --
  // [error word][counters][log2-sum-exp][O partials] -- fits; else one CTA per
  // segment (grid partition with a single split), which writes no partials
  atlas::DecodeLaunch L = atlas::plan_decode(batch, num_q_heads, num_kv_heads, q_len,
                                             max_seq_len, sms, 0, 0, atlas::kPartitionAuto);
  atlas::decode_fp8_fit_grid(head_dim, R < L.rows_per_cta ? R : L.rows_per_cta, sms, L);
  size_t counters_off = kAlign;
  size_t lse_off = counters_off + align_up((size_t)L.segs * sizeof(int32_t), kAlign);
  const size_t rows = (size_t)L.slots * L.rows_per_cta;
  size_t o_off = lse_off + align_up(rows * sizeof(float), kAlign);
  size_t clear = lse_off;  // error word + counters
  if (o_off + rows * head_dim * sizeof(float) > kScratchBytes) {
    const int whole = (int)(((long long)max_seq_len + 63) / 64 * 64);
    // one segment's unit table lives in shared memory: bound its length
    if (whole > kMaxWholeSegmentTokens) return ATLAS_ERR_WORKSPACE;
    L = atlas::plan_decode(batch, num_q_heads, num_kv_heads, q_len, max_seq_len, sms, whole, 0,
                           atlas::kPartitionGrid);
    lse_off = o_off = counters_off;
    clear = kAlign;
  }
  if (L.grid > 0x7FFFFFFFLL) return ATLAS_ERR_UNSUPPORTED;

  uint8_t* scratch = static_cast<uint8_t*>(scratch_on_current_device());
  if (!scratch) return ATLAS_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, clear, s) != cudaSuccess) return ATLAS_ERR_CUDA;

  atlas::DecodeParams p{};  // value-initialised: no fused append unless set
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k_pages = static_cast<const uint8_t*>(k_pages);
  p.v_pages = static_cast<const uint8_t*>(v_pages);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = reinterpret_cast<int32_t*>(scratch);
  p.counters = reinterpret_cast<int32_t*>(scratch + counters_off);
  p.part_lse = reinterpret_cast<float*>(scratch + lse_off);
  p.part_o = reinterpret_cast<float*>(scratch + o_off);
  p.B = batch;
  p.Hq = num_q_heads;
  p.Hkv = num_kv_heads;
  p.G = num_q_heads / num_kv_heads;
  p.q_len = q_len;
  p.D = head_dim;
  p.ps = page_size;
  p.num_pages = num_pages;
  p.max_blocks = max_blocks_per_seq;
  p.max_seq_len = max_seq_len;
  p.row_blocks = L.row_blocks;
  p.max_units = L.max_units;
  p.max_portions = L.max_portions;
  p.grid_mode = L.grid_mode;
  p.num_splits = L.num_splits;
  p.split_tokens = L.split_tokens;
  const double scale = sm_scale > 0.f ? (double)sm_scale : 1.0 / sqrt((double)head_dim);
  p.qk_scale_log2 = (float)(scale * 1.4426950408889634);  // log2(e)
  p.k_new = nullptr;  // decode only
  p.v_new = nullptr;
  p.wait_limit_ns = atlas::kDefaultWaitLimitNs;
  p.test_skip_unit = -1;
  cudaError_t e = atlas::launch_decode_fp8(p, L.rows_per_warp, L.rbg, L.stages, L.grid, s);
  return e == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}
