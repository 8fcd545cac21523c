// Host-side interfaces between the C ABI (api.cu) and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dsa.h"

namespace dsa {

constexpr int kPage = 64;
constexpr int kKeyTile = 128;     // keys per indexer MMA tile (M = 128)
constexpr int kRunTokens = 4;     // query tokens sharing one indexer key tile
constexpr int kMaxTopK = 2048;

void count_launch();
int num_sms();
// Pending test injection (see dsa_debug_inject); take_injection() consumes it.
int take_injection(int which);

// Launch `kernel` on `stream` with programmatic stream serialisation (the kernel may
// overlap the tail of the previous kernel in the stream; it must call pdl_wait()).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  count_launch();
  return e;
}

// ---- context-parallel decode ----------------------------------------------------------
size_t cp_merge_ws_bytes(int32_t T, int32_t G, int32_t k);
cudaError_t launch_cp_candidates(const float* logits, int64_t ld, int32_t T, const int32_t* idx,
                                 int32_t k, int32_t offset, float* values, int32_t* positions,
                                 cudaStream_t stream);
cudaError_t launch_cp_merge(const float* values, const int32_t* positions, int32_t G, int32_t T,
                            int32_t k, int32_t* idx_out, int32_t local_begin, int32_t local_end,
                            int32_t* idx_local, void* ws, cudaStream_t stream);
cudaError_t launch_cp_attn_merge(const uint16_t* o_parts, const float* lse_parts, int32_t G,
                                 int32_t T, int32_t H, int32_t d_v, uint16_t* out, float* lse,
                                 cudaStream_t stream);

// ---- cache append -------------------------------------------------------------------
cudaError_t launch_cache_append(const dsa_paged_cache* c, uint8_t* k8, float* k_scale,
                                uint16_t* kv, int32_t n_new, const int32_t* tok_seq,
                                const int32_t* tok_pos, const float* k_in, const uint16_t* kv_in,
                                cudaStream_t stream);

// ---- indexer ------------------------------------------------------------------------
size_t indexer_ws_bytes(int32_t n_tokens);
struct IndexerLaunch {
  const dsa_paged_cache* cache;
  const dsa_queries* queries;
  const uint8_t* q8;
  const float* q_scale;
  const float* w;
  int32_t n_idx_heads;
  float* logits;
  int64_t ld_logits;
  void* ws;
  cudaStream_t stream;
  uint32_t* hist = nullptr;     // optional [T][2048] first-digit histogram of the logits
  uint32_t* zero = nullptr;     // region the prep kernel zeroes first (histogram, counters)
  int64_t zero_words = 0;
  // query tokens with tok_pos < skip_below get no logits (the forward selects all of their
  // keys without reading any); 0: every token is scored
  int32_t skip_below = 0;
};
cudaError_t launch_indexer(const IndexerLaunch& a);

// ---- top-k --------------------------------------------------------------------------
size_t topk_ws_bytes(int32_t n_tokens, int32_t max_pos, int32_t k);
cudaError_t launch_topk(const float* logits, int64_t ld, const dsa_queries* q, int32_t k,
                        int32_t* idx, void* ws, cudaStream_t stream);
// decode variant: several CTAs per row, first digit from the indexer's histogram
struct TopkDecodeLayout {
  uint32_t* hist;
  uint32_t* arrive;
  int64_t zero_words;  // hist + arrive, from the start of the region
  int32_t* counts;
  int32_t* scr_a;
  int2* scr_b;
};
size_t topk_decode_ws_bytes(int32_t T, int64_t ld, int chunks);
int topk_decode_chunks(int32_t T, int32_t max_pos);
TopkDecodeLayout topk_decode_layout(void* ws, int32_t T, int64_t ld, int chunks);
cudaError_t launch_topk_decode(const float* logits, int64_t ld, const dsa_queries* q, int32_t k,
                               int32_t* idx, const TopkDecodeLayout& L, int chunks,
                               cudaStream_t stream);

// ---- sparse MLA attention --------------------------------------------------------------
size_t attn_ws_bytes(int32_t n_tokens, int32_t n_heads, int32_t d_v, int32_t k);
struct AttnLaunch {
  const dsa_paged_cache* cache;
  const dsa_queries* queries;
  const uint16_t* q;
  int32_t n_heads;
  int32_t d_v;
  float scale;
  const int32_t* idx;
  int32_t k;
  uint16_t* out;
  float* lse;
  void* ws;
  cudaStream_t stream;
};
cudaError_t launch_attn(const AttnLaunch& a);

// ---- status word ------------------------------------------------------------------------
cudaError_t read_and_clear_status(cudaStream_t stream, uint32_t* out);

}  // namespace dsa
