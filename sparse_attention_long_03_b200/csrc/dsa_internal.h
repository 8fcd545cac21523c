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
};
cudaError_t launch_indexer(const IndexerLaunch& a);

// ---- top-k --------------------------------------------------------------------------
size_t topk_ws_bytes(int32_t n_tokens, int32_t max_pos, int32_t k);
cudaError_t launch_topk(const float* logits, int64_t ld, const dsa_queries* q, int32_t k,
                        int32_t* idx, void* ws, cudaStream_t stream);

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
