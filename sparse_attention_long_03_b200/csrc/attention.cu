// Sparse MLA attention in MQA mode (DSA step 3) on sm_100a.
//
// "DeepSeek V3.2-Exp Cuts Prolonged-Context Costs ...", section "FP8 index -> top-k
// selection -> sparse core attention": item (2) runs standard attention over only the
// selected key-value entries; "Instantiation": MLA in MQA mode, every latent KV entry is
// shared by all query heads.  For query token t with selected positions S_t:
//   z[h,s] = scale * q[t,h,:] . kv[s,:]          (576 = 512 latent + 64 rope)
//   O[t,h,:] = sum_s softmax_s(z[h,s]) * kv[s,:512],   LSE[t,h] = log sum_s exp z[h,s]
//
// B200 design.  Heads sit on the MMA M dimension (128 rows), so each softmax thread owns
// one head row.  The full O (128 heads x 512 fp32) would fill all of TMEM, so a CLUSTER
// OF TWO CTAs shares one (token, key split):
//   * CTA 0 owns latent dims [0,256) + the rope dims, CTA 1 owns [256,512);
//   * each CTA computes its partial scores S_r = Q[:,own] . KV[:,own]^T (tcgen05, BF16,
//     fp32 in TMEM), the pair swaps partials through distributed shared memory and
//     both form S = S_0 + S_1 — no score FLOP is done twice and every latent byte is
//     read once;
//   * both run the identical online softmax; each accumulates O[:, own value dims] in
//     its own TMEM (256 columns) with P . V (P: bf16 in shared memory, A operand; V: the
//     gathered rows as an MN-major B operand — the same tiles the score MMA read).
// Selected rows are gathered with cp.async (16 B, manual 128-byte swizzle) through a
// two-stage ring.  Rescaling of O is lazy: the running max used for P only moves when it
// grows by more than 2^8, so O is rarely touched.  Long selections are split over several
// clusters (split-KV); a combine kernel merges the partial results by their LSE.
//
//   warp 0      producer: Q (once) and the selected latent rows, cp.async + mbarrier
//   warp 1      one thread issues tcgen05.mma for S and for P.V, and the commits
//   warps 2..5  softmax: partial-score exchange, online softmax, P, O rescale, output
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace attn {
constexpr int kBN = 64;            // keys per tile
constexpr int kMaxQC = 5;          // 64-dim chunks owned by one CTA (576 = 4*64 + 64 + 4*64)
constexpr int kQChunk = 128 * 128; // 128 heads x 64 bf16
constexpr int kKVChunk = kBN * 128;
constexpr int kKVStage = kMaxQC * kKVChunk;
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kMaxQC * kQChunk;
constexpr int kOffP = kOffKV + 2 * kKVStage;
constexpr int kOffX = kOffP + 128 * 128;
constexpr int kOffBar = kOffX + 128 * kBN * 4;
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 16;
constexpr int kSmemAlloc = kSmem + 1024;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
}  // namespace attn

struct AttnArgs {
  const uint16_t* q;
  const uint16_t* kv;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t num_blocks;
  const int32_t* tok_seq;
  const int32_t* tok_pos;
  const int32_t* idx;
  int32_t k;
  int32_t H;
  int32_t d_kv;
  int32_t d_v;
  float scale_log2;  // scale * log2(e)
  int32_t splits;
  int32_t per_split;  // selected slots per split (multiple of kBN)
  uint16_t* out;
  float* lse;
  float* part_o;    // [T, splits, H, d_v] fp32 (splits > 1)
  float* part_lse;  // [T, splits, H]
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitBudgetNs) return false;
  return true;
}

// Physical cache row of selected entry v of token t, or -1 if v is empty or invalid.
__device__ __forceinline__ int resolve_row(int v, int pos, int seq, const AttnArgs& a,
                                           bool report) {
  if (v < 0) return -1;
  if (v > pos) {
    if (report) record_error(kErrBadIndex);
    return -1;
  }
  const int p = a.block_table[static_cast<size_t>(seq) * a.max_blocks + v / kPage];
  if (p < 0 || p >= a.num_blocks) {
    if (report) record_error(kErrBadIndex);
    return -1;
  }
  return p * kPage + v % kPage;
}

struct ChunkPlan {
  int nq;         // chunks owned (score dims)
  int nvo;        // of which value chunks (the first nvo entries)
  int first_val;  // first owned value chunk
  int list[attn::kMaxQC];
};
__device__ __forceinline__ ChunkPlan chunk_plan(int d_kv, int d_v, int rank) {
  ChunkPlan c;
  const int nc = (d_kv + 63) / 64, nv = d_v / 64, nv0 = (nv + 1) / 2;
  c.nq = 0;
  if (rank == 0) {
    c.first_val = 0;
    c.nvo = nv0;
    for (int i = 0; i < nv0; ++i) c.list[c.nq++] = i;
    for (int i = nv; i < nc; ++i) c.list[c.nq++] = i;
  } else {
    c.first_val = nv0;
    c.nvo = nv - nv0;
    for (int i = nv0; i < nv; ++i) c.list[c.nq++] = i;
  }
  return c;
}

__global__ void __launch_bounds__(192, 1) __cluster_dims__(2, 1, 1)
    sparse_mla_kernel(const AttnArgs a) {
  using namespace attn;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;   // [2]
  uint64_t* kv_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;    // [2]
  uint64_t* s_free = bars + 7;    // [2]
  uint64_t* p_full = bars + 9;
  uint64_t* pv_done = bars + 10;
  uint64_t* x_full = bars + 11;  // peer wrote its partial scores into my X
  uint64_t* x_free = bars + 12;  // peer consumed the partial I wrote into its X
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const uint32_t peer = rank ^ 1u;
  const int t = blockIdx.y;
  const int split = blockIdx.x >> 1;
  const ChunkPlan cp = chunk_plan(a.d_kv, a.d_v, static_cast<int>(rank));
  const int seq = a.tok_seq[t];
  const int pos = a.tok_pos[t];
  const int k0 = split * a.per_split;
  const int k1 = min(a.k, k0 + a.per_split);
  const int n_tiles = k1 > k0 ? (k1 - k0 + kBN - 1) / kBN : 0;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 32);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 32);
      mbar_init(&kv_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(x_full, 128);
    mbar_init(x_free, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers are initialised before anyone arrives remotely
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_o = tmem + 2 * kBN;

  uint8_t* qs = smem + kOffQ;
  uint8_t* kvs = smem + kOffKV;
  uint8_t* ps = smem + kOffP;
  float* xs = reinterpret_cast<float*>(smem + kOffX);

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    // Q: own chunks, 128 rows (heads >= H are zero), 8 x 16 B per row and chunk
    for (int p = lane; p < cp.nq * 128 * 8; p += 32) {
      const int oc = p / (128 * 8), rem = p % (128 * 8), h = rem / 8, c16 = rem % 8;
      const int d0 = cp.list[oc] * 64 + c16 * 8;  // first element of this 16-byte piece
      const int valid = (h < a.H) ? max(0, min(8, a.d_kv - d0)) : 0;
      const uint16_t* src = valid ? a.q + (static_cast<size_t>(t) * a.H + h) * a.d_kv + d0 : a.q;
      cp_async_16(qs + oc * kQChunk + swz_offset(h, c16 * 16, 128), src, valid * 2);
    }
    cp_async_arrive_noinc(q_full);
    pdl_wait();  // the selection comes from the previous kernel
    int i = 0;
    for (; i < n_tiles; ++i) {
      const int st = i & 1;
      if (!mbar_wait(&kv_empty[st], ((i >> 1) & 1) ^ 1, abort_flag)) break;
      // resolve the 64 rows of this tile: lane handles slots lane and lane + 32
      int rows[2];
      for (int u = 0; u < 2; ++u) {
        const int slot = k0 + i * kBN + lane + 32 * u;
        const int v = slot < k1 ? a.idx[static_cast<size_t>(t) * a.k + slot] : -1;
        rows[u] = resolve_row(v, pos, seq, a, true);
      }
      uint8_t* dst_stage = kvs + st * kKVStage;
      for (int p = lane; p < kBN * cp.nq * 8; p += 32) {
        const int slot = p / (cp.nq * 8), rem = p % (cp.nq * 8), oc = rem / 8, c16 = rem % 8;
        const int r0 = __shfl_sync(0xffffffffu, rows[0], slot & 31);
        const int r1 = __shfl_sync(0xffffffffu, rows[1], slot & 31);
        const int row = (slot >> 5) ? r1 : r0;
        const int d0 = cp.list[oc] * 64 + c16 * 8;
        const int valid = row >= 0 ? max(0, min(8, a.d_kv - d0)) : 0;
        const uint16_t* src = valid ? a.kv + static_cast<size_t>(row) * a.d_kv + d0 : a.kv;
        cp_async_16(dst_stage + oc * kKVChunk + swz_offset(slot, c16 * 16, 128), src, valid * 2);
      }
      cp_async_arrive_noinc(&kv_full[st]);
    }
    cp_async_wait<0>();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    pdl_wait();
    if (lane == 0) {
      const uint32_t idesc_s = instr_desc(128, kBN, 1, 1, 0, 0);
      const uint32_t idesc_pv = instr_desc(128, cp.nvo > 0 ? cp.nvo * 64 : 64, 1, 1, 0, 1);
      const uint32_t q_base = smem_u32(qs), kv_base = smem_u32(kvs), p_base = smem_u32(ps);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      auto do_pv = [&](int j) -> bool {
        if (!mbar_wait(p_full, j & 1, abort_flag)) return false;
        tc_fence_after();
        fence_proxy_async_smem();
        if (cp.nvo > 0) {
          const uint32_t vb = kv_base + (j & 1) * kKVStage;
#pragma unroll
          for (int ks = 0; ks < kBN / 16; ++ks)
            mma_bf16(tmem_o, smem_desc(p_base + ks * 32, 16, 1024, kSw128),
                     smem_desc(vb + ks * 2048, kKVChunk, 1024, kSw128), idesc_pv,
                     (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[j & 1]);
        mma_commit(pv_done);
        return true;
      };
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int st = i & 1;
        if (!mbar_wait(&kv_full[st], (i >> 1) & 1, abort_flag)) break;
        if (!mbar_wait(&s_free[st], ((i >> 1) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        fence_proxy_async_smem();
        const uint32_t kb = kv_base + st * kKVStage;
        bool first = true;
        for (int oc = 0; oc < cp.nq; ++oc) {
          const int w = min(64, a.d_kv - cp.list[oc] * 64);
          for (int ks = 0; ks < (w + 15) / 16; ++ks) {
            mma_bf16(tmem + st * kBN, smem_desc(q_base + oc * kQChunk + ks * 32, 16, 1024, kSw128),
                     smem_desc(kb + oc * kKVChunk + ks * 32, 16, 1024, kSw128), idesc_s,
                     first ? 0u : 1u);
            first = false;
          }
        }
        mma_commit(&s_full[st]);
        if (i > 0 && !do_pv(i - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && n_tiles > 0) do_pv(n_tiles - 1);
      mma_commit(drain);
      wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax (warps 2..5)
    const int quarter = warp & 3;
    const int h = quarter * 32 + lane;  // head row == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t x_peer = map_peer(smem_u32(xs + h * kBN), peer);
    pdl_wait();
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i & 1;
      // validity of the tile's 64 slots (same rule as the producer)
      uint32_t vm[2];
      for (int u = 0; u < 2; ++u) {
        const int slot = k0 + i * kBN + lane + 32 * u;
        const int v = slot < k1 ? a.idx[static_cast<size_t>(t) * a.k + slot] : -1;
        vm[u] = __ballot_sync(0xffffffffu, resolve_row(v, pos, seq, a, false) >= 0);
      }
      if (!mbar_wait(&s_full[st], (i >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
      if (cp.nq > 0) {
        tmem_ld32(tmem + lane_off + st * kBN, s);
        tmem_ld32(tmem + lane_off + st * kBN + 32, s + 32);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < kBN; ++j) s[j] = 0.f;
      }
      tc_fence_before();
      mbar_arrive(&s_free[st]);
      // swap partial scores with the peer CTA
      if (i > 0 && !mbar_wait_cluster(x_free, (i - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int c = 0; c < kBN / 4; ++c) {
        const int slot4 = (c + h) & (kBN / 4 - 1);
        st_cluster_v4(x_peer + slot4 * 16, s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
      }
      mbar_arrive_cluster(x_full, peer);
      if (!mbar_wait_cluster(x_full, i & 1, abort_flag)) {
        ok = false;
        break;
      }
      const float4* xr = reinterpret_cast<const float4*>(xs + h * kBN);
#pragma unroll
      for (int c = 0; c < kBN / 4; ++c) {
        const float4 o = xr[(c + h) & (kBN / 4 - 1)];
        // S = S_rank0 + S_rank1 in the same order on both CTAs
        if (rank == 0) {
          s[4 * c] += o.x;
          s[4 * c + 1] += o.y;
          s[4 * c + 2] += o.z;
          s[4 * c + 3] += o.w;
        } else {
          s[4 * c] = o.x + s[4 * c];
          s[4 * c + 1] = o.y + s[4 * c + 1];
          s[4 * c + 2] = o.z + s[4 * c + 2];
          s[4 * c + 3] = o.w + s[4 * c + 3];
        }
      }
      mbar_arrive_cluster(x_free, peer);
      // online softmax in log2 units
      float m_tile = -INFINITY;
#pragma unroll
      for (int j = 0; j < kBN; ++j) {
        const bool valid = (vm[j >> 5] >> (j & 31)) & 1u;
        s[j] = valid ? s[j] * a.scale_log2 : -INFINITY;
        m_tile = fmaxf(m_tile, s[j]);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (m_used == -INFINITY) {
        m_used = m_tile;
      } else if (m_tile > m_used + kRescaleThreshold) {
        alpha = exp2f(m_used - m_tile);
        m_used = m_tile;
        rescale = true;
      }
      uint32_t pk[kBN / 2];
      float psum = 0.f;
#pragma unroll
      for (int j = 0; j < kBN; j += 2) {
        const float p0 = s[j] == -INFINITY ? 0.f : exp2f(s[j] - m_used);
        const float p1 = s[j + 1] == -INFINITY ? 0.f : exp2f(s[j + 1] - m_used);
        pk[j / 2] = pack_bf16x2(p0, p1);
        const float r0 = __uint_as_float(pk[j / 2] << 16);
        const float r1 = __uint_as_float(pk[j / 2] & 0xFFFF0000u);
        psum += r0 + r1;
      }
      // P buffer and O are free once the previous P.V has completed
      if (i > 0 && !mbar_wait(pv_done, (i - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (rescale && cp.nvo > 0) {
        for (int c = 0; c < cp.nvo * 64; c += 32) {
          float o[32];
          tmem_ld32(tmem_o + lane_off + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] *= alpha;
          tmem_st32(tmem_o + lane_off + c, o);
        }
        tmem_wait_st();
      }
      l = l * alpha + psum;
#pragma unroll
      for (int c = 0; c < kBN / 8; ++c) {
        uint4 v = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(ps + swz_offset(h, c * 16, 128)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (ok && n_tiles > 0 && !mbar_wait(pv_done, (n_tiles - 1) & 1, abort_flag)) ok = false;
    tc_fence_after();
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const float lse_val = l > 0.f ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    const int vbase = cp.first_val * 64;
    if (a.splits == 1) {
      if (ok && cp.nvo > 0) {
        for (int c = 0; c < cp.nvo * 64; c += 32) {
          float o[32];
          if (n_tiles > 0) {
            tmem_ld32(tmem_o + lane_off + c, o);
            tmem_wait_ld();
          }
          if (h < a.H) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = n_tiles > 0 ? pack_bf16x2(o[2 * j] * inv_l, o[2 * j + 1] * inv_l) : 0u;
            uint4* dst = reinterpret_cast<uint4*>(
                a.out + (static_cast<size_t>(t) * a.H + h) * a.d_v + vbase + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
      }
      if (rank == 0 && h < a.H && a.lse) a.lse[static_cast<size_t>(t) * a.H + h] = lse_val;
    } else {
      const size_t row = (static_cast<size_t>(t) * a.splits + split) * a.H + h;
      if (ok && cp.nvo > 0 && h < a.H) {
        for (int c = 0; c < cp.nvo * 64; c += 32) {
          float o[32];
          if (n_tiles > 0) {
            tmem_ld32(tmem_o + lane_off + c, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0.f;
          }
          float4* dst = reinterpret_cast<float4*>(a.part_o + row * a.d_v + vbase + c);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(o[4 * j] * inv_l, o[4 * j + 1] * inv_l, o[4 * j + 2] * inv_l,
                                 o[4 * j + 3] * inv_l);
        }
      }
      if (rank == 0 && h < a.H) a.part_lse[row] = lse_val;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still touch its shared memory
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge split-KV partial results: O = sum_s exp(lse_s - LSE) O_s, LSE = logsumexp_s lse_s.
__global__ void __launch_bounds__(128) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse,
                                                           int splits, int H, int d_v,
                                                           uint16_t* __restrict__ out,
                                                           float* __restrict__ lse) {
  const int t = blockIdx.y, h = blockIdx.x;
  __shared__ float wsh[64];
  __shared__ float lse_sh;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < 32) {
    float m = -INFINITY;
    for (int s = threadIdx.x; s < splits; s += 32)
      m = fmaxf(m, part_lse[(static_cast<size_t>(t) * splits + s) * H + h]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
    for (int s = threadIdx.x; s < splits; s += 32) {
      const float ls = part_lse[(static_cast<size_t>(t) * splits + s) * H + h];
      const float e = (m == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - m);
      wsh[s] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = sum > 0.f ? 1.f / sum : 0.f;
    for (int s = threadIdx.x; s < splits; s += 32) wsh[s] *= inv;
    if (threadIdx.x == 0) lse_sh = sum > 0.f ? m + __logf(sum) : -INFINITY;
  }
  __syncthreads();
  for (int d = threadIdx.x * 4; d < d_v; d += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < splits; ++s) {
      const float w = wsh[s];
      if (w == 0.f) continue;
      const float4 v = *reinterpret_cast<const float4*>(
          part_o + ((static_cast<size_t>(t) * splits + s) * H + h) * d_v + d);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    *reinterpret_cast<uint2*>(out + (static_cast<size_t>(t) * H + h) * d_v + d) = pk;
  }
  if (threadIdx.x == 0 && lse) lse[static_cast<size_t>(t) * H + h] = lse_sh;
}

// ---------------------------------------------------------------------------- host
static int attn_splits(int T, int k) {
  const int tiles = (k + attn::kBN - 1) / attn::kBN;
  const int clusters = num_sms() / 2;
  int want = T > 0 ? clusters / T : 1;
  if (want < 1) want = 1;
  if (want > tiles) want = tiles;
  if (want > 64) want = 64;
  int per_tiles = (tiles + want - 1) / want;
  return (tiles + per_tiles - 1) / per_tiles;
}

size_t attn_ws_bytes(int32_t T, int32_t H, int32_t d_v, int32_t k) {
  if (T <= 0) return 0;
  const int splits = attn_splits(T, k);
  if (splits <= 1) return 0;
  const size_t o = static_cast<size_t>(T) * splits * H * d_v * 4;
  const size_t l = static_cast<size_t>(T) * splits * H * 4;
  return ((o + 255) & ~static_cast<size_t>(255)) + ((l + 255) & ~static_cast<size_t>(255));
}

cudaError_t launch_attn(const AttnLaunch& L) {
  const int T = L.queries->n_tokens;
  if (T == 0) return cudaSuccess;
  static int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(sparse_mla_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         attn::kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  const int tiles = (L.k + attn::kBN - 1) / attn::kBN;
  const int splits = attn_splits(T, L.k);
  const int per_tiles = (tiles + splits - 1) / splits;
  AttnArgs a;
  a.q = L.q;
  a.kv = L.cache->kv;
  a.block_table = L.cache->block_table;
  a.max_blocks = L.cache->max_blocks_per_seq;
  a.num_blocks = L.cache->num_blocks;
  a.tok_seq = L.queries->tok_seq;
  a.tok_pos = L.queries->tok_pos;
  a.idx = L.idx;
  a.k = L.k;
  a.H = L.n_heads;
  a.d_kv = L.cache->d_kv;
  a.d_v = L.d_v;
  a.scale_log2 = L.scale * attn::kLog2e;
  a.splits = splits;
  a.per_split = per_tiles * attn::kBN;
  a.out = L.out;
  a.lse = L.lse;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  if (splits > 1) {
    const size_t o = static_cast<size_t>(T) * splits * L.n_heads * L.d_v * 4;
    a.part_o = static_cast<float*>(L.ws);
    a.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(L.ws) +
                                          ((o + 255) & ~static_cast<size_t>(255)));
  }
  cudaError_t e = launch_pdl(sparse_mla_kernel, dim3(2 * splits, T), dim3(192), attn::kSmemAlloc,
                             L.stream, a);
  if (e != cudaSuccess || splits == 1) return e;
  return launch_pdl(attn_combine_kernel, dim3(L.n_heads, T), dim3(128), 0, L.stream, a.part_o,
                    a.part_lse, splits, L.n_heads, L.d_v, L.out, L.lse);
}

}  // namespace dsa
