// Cache append: the step that fills the paged caches the DSA path reads.
//
// "DeepSeek V3.2-Exp: Sparse Attention, Long Context, and Cheaper API" (sections "Quick
// guide to run it locally" and "Open kernels") has the caches paged in 64-token blocks;
// "DeepSeek V3.2-Exp Cuts Prolonged-Context Costs ...", section "FP8 index -> top-k
// selection -> sparse core attention", has the index keys in FP8.  Each new token's index
// key is quantised with one fp32 scale per token, s = amax / 448 (1 if amax = 0), and
// codes e4m3(key / s) rounded to nearest even and saturating at 448; its latent row is
// copied as is.
//
// One warp per token: the key's absolute maximum by a warp reduction, then every lane
// converts four elements at a time and writes them as one 32-bit store; the latent row
// moves in 16-byte pieces.  Plain loads and stores: a token's data is a few hundred bytes.
#include <cuda_fp8.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

struct AppendArgs {
  uint8_t* k8;
  float* k_scale;
  uint16_t* kv;
  const int32_t* block_table;
  int32_t batch;
  int32_t max_blocks;
  int32_t num_blocks;
  int32_t idx_dim;
  int32_t d_kv;
  int32_t n_new;
  const int32_t* tok_seq;
  const int32_t* tok_pos;
  const float* k_in;
  const uint16_t* kv_in;
};

constexpr int kAppendWarps = 8;

__global__ void __launch_bounds__(kAppendWarps * 32) cache_append_kernel(const AppendArgs a) {
  pdl_wait();  // the new keys may come from the kernel before
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
  if (i >= a.n_new) return;
  const int b = a.tok_seq[i], pos = a.tok_pos[i];
  if (b < 0 || b >= a.batch || pos < 0 || pos >= a.max_blocks * kPage) {
    if (lane == 0) record_error(kErrBadIndex);
    return;
  }
  const int blk = a.block_table[static_cast<size_t>(b) * a.max_blocks + pos / kPage];
  if (blk < 0 || blk >= a.num_blocks) {
    if (lane == 0) record_error(kErrBadIndex);
    return;
  }
  const size_t row = static_cast<size_t>(blk) * kPage + pos % kPage;

  const float4* key = reinterpret_cast<const float4*>(a.k_in + static_cast<size_t>(i) * a.idx_dim);
  const int n4 = a.idx_dim / 4;
  float amax = 0.f;
  for (int e = lane; e < n4; e += 32) {
    const float4 v = key[e];
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = amax > 0.f ? amax / 448.f : 1.f;
  uint32_t* dst = reinterpret_cast<uint32_t*>(a.k8 + row * a.idx_dim);
  for (int e = lane; e < n4; e += 32) {
    const float4 v = key[e];
    const uint32_t c0 = __nv_cvt_float_to_fp8(v.x / s, __NV_SATFINITE, __NV_E4M3);
    const uint32_t c1 = __nv_cvt_float_to_fp8(v.y / s, __NV_SATFINITE, __NV_E4M3);
    const uint32_t c2 = __nv_cvt_float_to_fp8(v.z / s, __NV_SATFINITE, __NV_E4M3);
    const uint32_t c3 = __nv_cvt_float_to_fp8(v.w / s, __NV_SATFINITE, __NV_E4M3);
    dst[e] = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
  }
  if (lane == 0) a.k_scale[row] = s;

  if (a.kv && a.kv_in) {
    const uint4* src = reinterpret_cast<const uint4*>(a.kv_in + static_cast<size_t>(i) * a.d_kv);
    uint4* out = reinterpret_cast<uint4*>(a.kv + row * a.d_kv);
    for (int e = lane; e < a.d_kv / 8; e += 32) out[e] = src[e];
  }
}

}  // namespace

cudaError_t launch_cache_append(const dsa_paged_cache* c, uint8_t* k8, float* k_scale,
                                uint16_t* kv, int32_t n_new, const int32_t* tok_seq,
                                const int32_t* tok_pos, const float* k_in, const uint16_t* kv_in,
                                cudaStream_t stream) {
  if (n_new == 0) return cudaSuccess;
  AppendArgs a{k8,       k_scale,   kv,    c->block_table, c->batch, c->max_blocks_per_seq,
               c->num_blocks, c->idx_dim, c->d_kv, n_new, tok_seq, tok_pos, k_in, kv_in};
  const int grid = (n_new + kAppendWarps - 1) / kAppendWarps;
  return launch_pdl(cache_append_kernel, dim3(grid), dim3(kAppendWarps * 32), 0, stream, a);
}

}  // namespace dsa
