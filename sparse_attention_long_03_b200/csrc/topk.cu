// Fine-grained token selection (DSA step 2): the k largest index logits of each query row.
//
// "DeepSeek V3.2-Exp Cuts Prolonged-Context Costs ...", section "FP8 index -> top-k
// selection -> sparse core attention", item (2): keep only the top-k (k = 2048) key
// entries per query.  Equal logits: the smaller position wins; fewer than k valid
// positions: all of them are selected.
//
// Radix select, no sort.  A logit becomes an order-preserving uint32 key (sign bit
// flipped for positives, all bits inverted for negatives).  Digits of 11, 11 and 10 bits
// are resolved from the top with shared-memory histograms (warp-aggregated atomics via
// __match_any_sync) and a block-wide suffix scan.  After the first digit every element of
// a higher bucket is already selected and is written out at once; the elements of the
// threshold bucket are gathered (in position order) into a shared candidate list, and
// the two remaining digits run on that list only.  All writes are ordered compactions
// (each thread classifies a run of consecutive elements, one block scan per round), so
// the result is deterministic.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCand = 8192;       // threshold-bucket candidates kept in shared memory
constexpr int kTopkRowCache = 32768;  // rows up to this length are cached in shared memory

constexpr int kTopkMaxChunks = 128;  // CTAs per row in the decode variant

struct TopkSmem {
  uint32_t hist[2048];
  int scan[72];
  int sel[4];
  int pre_a[kTopkMaxChunks + 1];
  int pre_b[kTopkMaxChunks + 1];
  uint32_t cand_key[kTopkCand];
  int32_t cand_idx[kTopkCand];
};
constexpr size_t kTopkSmemBase = sizeof(TopkSmem);
constexpr size_t kTopkSmemMax = kTopkSmemBase + kTopkRowCache * sizeof(uint32_t);

size_t topk_ws_bytes(int32_t, int32_t, int32_t) { return 0; }

struct RowGlobal {
  const float* row;
  __device__ uint32_t key(int i) const { return float_to_ordered(row[i]); }
  __device__ int index(int i) const { return i; }
};
struct RowGlobalOff {
  const float* row;
  int off;
  __device__ uint32_t key(int i) const { return float_to_ordered(row[off + i]); }
  __device__ int index(int i) const { return off + i; }
};
struct CandGlobal {
  const float* row;
  const int32_t* list;
  __device__ uint32_t key(int i) const { return float_to_ordered(row[list[i]]); }
  __device__ int index(int i) const { return list[i]; }
};
struct RowCachedOff {
  const uint32_t* keys;
  int off;
  __device__ uint32_t key(int i) const { return keys[i]; }
  __device__ int index(int i) const { return off + i; }
};
struct RowCached {
  const uint32_t* keys;
  __device__ uint32_t key(int i) const { return keys[i]; }
  __device__ int index(int i) const { return i; }
};
struct RowCand {
  const uint32_t* keys;
  const int32_t* idx;
  __device__ uint32_t key(int i) const { return keys[i]; }
  __device__ int index(int i) const { return idx[i]; }
};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Block-wide exclusive scan of two counters per warp (warp totals in sm->scan).
// Returns per-warp exclusive offsets for class A and class B and the block totals.
__device__ __forceinline__ void scan_two(TopkSmem* sm, int wa, int wb, int* off_a, int* off_b,
                                         int* tot_a, int* tot_b) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) {
    sm->scan[wid] = wa;
    sm->scan[32 + wid] = wb;
  }
  __syncthreads();
  if (wid == 0) {
    const bool live = lane < static_cast<int>(blockDim.x >> 5);
    int a = live ? sm->scan[lane] : 0, b = live ? sm->scan[32 + lane] : 0;
    int ia = a, ib = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, ia, o), yb = __shfl_up_sync(0xffffffffu, ib, o);
      if (lane >= o) {
        ia += ya;
        ib += yb;
      }
    }
    sm->scan[lane] = ia - a;
    sm->scan[32 + lane] = ib - b;
    if (lane == 31) {
      sm->scan[64] = ia;
      sm->scan[65] = ib;
    }
  }
  __syncthreads();
  *off_a = sm->scan[wid];
  *off_b = sm->scan[32 + wid];
  *tot_a = sm->scan[64];
  *tot_b = sm->scan[65];
  __syncthreads();
}

// Histogram of digit = (key >> shift) & (nb-1) over elements with (key >> pshift) == prefix
// (pshift == 32: every element).
template <class Src>
__device__ void hist_pass(TopkSmem* sm, const Src& src, int n, int shift, int nb, int pshift,
                          uint32_t prefix) {
  for (int b = threadIdx.x; b < 2048; b += blockDim.x) sm->hist[b] = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    bool take = false;
    uint32_t d = 0;
    if (i < n) {
      const uint32_t k = src.key(i);
      take = pshift >= 32 || (k >> pshift) == prefix;
      d = (k >> shift) & static_cast<uint32_t>(nb - 1);
    }
    const uint32_t active = __ballot_sync(0xffffffffu, take);
    if (take) {
      const uint32_t peers = __match_any_sync(active, d);
      if ((lanemask_lt() & peers) == 0) atomicAdd(&sm->hist[d], __popc(peers));
    }
  }
  __syncthreads();
}

// Largest bucket b with count(> b) < k_rem <= count(>= b).  Writes sel[0] = b,
// sel[1] = count(> b), sel[2] = count(b).  Thread t looks at `per` consecutive buckets in
// descending order, starting at nb-1-t*per.
__device__ void select_bucket(TopkSmem* sm, int nb, int k_rem) {
  const int t = threadIdx.x;
  const int per = (nb + blockDim.x - 1) / blockDim.x;  // 1, 2 or 4
  int c[4];
  int sum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int b = nb - 1 - t * per - q;
    c[q] = (q < per && b >= 0) ? static_cast<int>(sm->hist[b]) : 0;
    sum += c[q];
  }
  const int lane = t & 31, wid = t >> 5;
  int x = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm->scan[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const int v = lane < static_cast<int>(blockDim.x >> 5) ? sm->scan[lane] : 0;
    int iv = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, iv, o);
      if (lane >= o) iv += y;
    }
    sm->scan[lane] = iv - v;
  }
  __syncthreads();
  int run = sm->scan[wid] + x - sum;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int b = nb - 1 - t * per - q;
    if (q < per && b >= 0 && run < k_rem && run + c[q] >= k_rem) {
      sm->sel[0] = b;
      sm->sel[1] = run;
      sm->sel[2] = c[q];
    }
    run += c[q];
  }
  __syncthreads();
}

// Block-wide exclusive scan of two per-thread counters.
__device__ __forceinline__ void thread_scan_two(TopkSmem* sm, int a, int b, int* off_a,
                                                int* off_b, int* tot_a, int* tot_b) {
  const int lane = threadIdx.x & 31;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, o), yb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += ya;
      ib += yb;
    }
  }
  int wa, wb, ta, tb;
  scan_two(sm, __shfl_sync(0xffffffffu, ia, 31), __shfl_sync(0xffffffffu, ib, 31), &wa, &wb, &ta,
           &tb);
  *off_a = wa + ia - a;
  *off_b = wb + ib - b;
  *tot_a = ta;
  *tot_b = tb;
}

// The same ordered compaction with one block scan per round of blockDim.x * E elements:
// thread t owns E consecutive elements (E odd, so a warp's shared-memory reads of its
// elements fall in 32 different banks), counts its two classes, and after the scan writes
// its elements in position order.
template <int E, class Src, class Cls, class SinkA, class SinkB>
__device__ int2 ordered_pass_seg(TopkSmem* sm, const Src& src, int n, Cls cls, SinkA sinkA,
                                 SinkB sinkB, int limitB) {
  static_assert(E % 2 == 1 && E <= 31, "odd element count per thread");
  int run_a = 0, run_b = 0;
  for (int base = 0; base < n; base += static_cast<int>(blockDim.x) * E) {
    const int i0 = base + static_cast<int>(threadIdx.x) * E;
    uint32_t keys[E];
    uint32_t ma = 0, mb = 0;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      keys[j] = 0;
      if (i0 + j < n) {
        keys[j] = src.key(i0 + j);
        const int c = cls(keys[j]);
        if (c == 1) ma |= 1u << j;
        if (c == 2) mb |= 1u << j;
      }
    }
    int off_a, off_b, tot_a, tot_b;
    thread_scan_two(sm, __popc(ma), __popc(mb), &off_a, &off_b, &tot_a, &tot_b);
    int ra = run_a + off_a, rb = run_b + off_b;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      if ((ma >> j) & 1u) sinkA(ra++, keys[j], src.index(i0 + j));
      if ((mb >> j) & 1u) {
        if (rb < limitB) sinkB(rb, keys[j], src.index(i0 + j));
        ++rb;
      }
    }
    run_a += tot_a;
    run_b += tot_b;
  }
  return make_int2(run_a, run_b);
}

// Digits 2 and 3 over the threshold-bucket candidates of digit-1 bucket b1, then the
// ordered output of the k2 entries they contribute, at out[0 .. k2).
template <class Src>
__device__ void finish_candidates(TopkSmem* sm, const Src& cs, int n_cand, uint32_t b1, int k2,
                                  int32_t* out) {
  hist_pass(sm, cs, n_cand, 10, 2048, 32, 0u);
  select_bucket(sm, 2048, k2);
  const uint32_t b2 = static_cast<uint32_t>(sm->sel[0]);
  const int above2 = sm->sel[1];
  hist_pass(sm, cs, n_cand, 0, 1024, 10, (b1 << 11) | b2);
  select_bucket(sm, 1024, k2 - above2);
  const uint32_t thr = (b1 << 21) | (b2 << 10) | static_cast<uint32_t>(sm->sel[0]);
  const int need_eq = k2 - above2 - sm->sel[1];
  int32_t* eq_out = out + (k2 - need_eq);
  ordered_pass_seg<3>(
      sm, cs, n_cand, [thr](uint32_t key) { return key > thr ? 1 : (key == thr ? 2 : 0); },
      [out](int r, uint32_t, int idx) { out[r] = idx; },
      [eq_out](int r, uint32_t, int idx) { eq_out[r] = idx; }, need_eq);
}

template <class Src>
__device__ void select_from(TopkSmem* sm, const Src& src, int n, int k, int32_t* out) {
  // digit 1: bits 21..31
  hist_pass(sm, src, n, 21, 2048, 32, 0u);
  select_bucket(sm, 2048, k);
  const uint32_t b1 = static_cast<uint32_t>(sm->sel[0]);
  const int above1 = sm->sel[1];
  const int n_cand = sm->sel[2];
  const int k2 = k - above1;
  if (n_cand <= kTopkCand) {
    // higher buckets are final; gather the threshold bucket in position order
    ordered_pass_seg<7>(
        sm, src, n,
        [b1](uint32_t key) { return (key >> 21) > b1 ? 1 : ((key >> 21) == b1 ? 2 : 0); },
        [out](int r, uint32_t, int idx) { out[r] = idx; },
        [sm](int r, uint32_t key, int idx) {
          sm->cand_key[r] = key;
          sm->cand_idx[r] = idx;
        },
        kTopkCand);
    __syncthreads();
    finish_candidates(sm, RowCand{sm->cand_key, sm->cand_idx}, n_cand, b1, k2, out + above1);
  } else {
    hist_pass(sm, src, n, 10, 2048, 21, b1);
    select_bucket(sm, 2048, k2);
    const uint32_t b2 = static_cast<uint32_t>(sm->sel[0]);
    const int above2 = sm->sel[1];
    hist_pass(sm, src, n, 0, 1024, 10, (b1 << 11) | b2);
    select_bucket(sm, 1024, k2 - above2);
    const uint32_t thr = (b1 << 21) | (b2 << 10) | static_cast<uint32_t>(sm->sel[0]);
    const int need_eq = k2 - above2 - sm->sel[1];
    int32_t* eq_out = out + (k - need_eq);
    ordered_pass_seg<7>(
        sm, src, n, [thr](uint32_t key) { return key > thr ? 1 : (key == thr ? 2 : 0); },
        [out](int r, uint32_t, int idx) { out[r] = idx; },
        [eq_out](int r, uint32_t, int idx) { eq_out[r] = idx; }, need_eq);
  }
}

__global__ void __launch_bounds__(kTopkThreads, 1)
    topk_kernel(const float* __restrict__ logits, int64_t ld, const int32_t* __restrict__ tok_pos,
                int32_t max_pos, int32_t k, int32_t* __restrict__ idx, int cache_ok) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem* sm = reinterpret_cast<TopkSmem*>(topk_smem_raw);
  uint32_t* row_cache = reinterpret_cast<uint32_t*>(topk_smem_raw + kTopkSmemBase);
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  int32_t* out = idx + static_cast<int64_t>(t) * k;
  const int pos = tok_pos[t];
  if (pos < 0 || pos > max_pos) {
    if (threadIdx.x == 0) record_error(kErrBadIndex);
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = -1;
    return;
  }
  const int n = pos + 1;
  const float* row = logits + static_cast<int64_t>(t) * ld;
  if (n <= k) {
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  if (cache_ok && n <= kTopkRowCache) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) row_cache[i] = float_to_ordered(row[i]);
    __syncthreads();
    select_from(sm, RowCached{row_cache}, n, k, out);
  } else {
    select_from(sm, RowGlobal{row}, n, k, out);
  }
}

cudaError_t launch_topk(const float* logits, int64_t ld, const dsa_queries* q, int32_t k,
                        int32_t* idx, void*, cudaStream_t stream) {
  if (q->n_tokens == 0) return cudaSuccess;
  const int cache_ok = (q->max_pos + 1) <= kTopkRowCache ? 1 : 0;
  const size_t smem = cache_ok ? kTopkSmemMax : kTopkSmemBase;
  static int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kTopkSmemMax));
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  return launch_pdl(topk_kernel, dim3(q->n_tokens), dim3(kTopkThreads), smem, stream, logits, ld,
                    q->tok_pos, q->max_pos, k, idx, cache_ok);
}

// ---------------------------------------------------------------------------- decode variant
// Few long rows (decode): the row is split over `chunks` CTAs.  The first radix digit comes
// from the histogram the indexer built while writing the logits, so every CTA knows the
// threshold bucket b1 at once.  Each CTA writes, in position order, its entries above b1
// (final) and its entries in b1 (candidates) to scratch at its own position range and
// posts the two counts; the last CTA to arrive (global counter, no waiting) concatenates
// the finals in chunk order and resolves digits 2 and 3 over the candidates.  Output order
// equals the single-CTA kernel's: finals ascending, then candidate winners ascending.
constexpr int kTopkDecThreads = 512;

struct TopkDecodeWs {
  const uint32_t* hist;  // [T][2048] digit-1 histogram (from the indexer epilogue)
  uint32_t* arrive;      // [T] arrival counters, zero on entry
  int32_t* counts;       // [T][chunks][2]
  int32_t* scr_a;        // [T][ld] finals, at each chunk's position range
  int2* scr_b;           // [T][ld] candidates (position, ordered key), same
};

// Threshold-bucket candidates read back by the finishing CTA: (position, key) pairs.
struct CandPairs {
  const int2* list;
  __device__ uint32_t key(int i) const { return static_cast<uint32_t>(list[i].y); }
  __device__ int index(int i) const { return list[i].x; }
};

__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}

// Chunk elements each thread classifies per round of the decode pass (odd, see
// ordered_pass_seg).
constexpr int kDecPerThread = 7;

__global__ void __launch_bounds__(kTopkDecThreads, 1)
    topk_decode_kernel(const float* __restrict__ logits, int64_t ld,
                       const int32_t* __restrict__ tok_pos, int32_t max_pos, int32_t k,
                       int32_t* __restrict__ idx, TopkDecodeWs ws, int chunks) {
  extern __shared__ uint8_t topk_smem_raw[];
  TopkSmem* sm = reinterpret_cast<TopkSmem*>(topk_smem_raw);
  pdl_wait();  // logits and histogram come from the indexer
  pdl_trigger();
  const int t = blockIdx.y, c = blockIdx.x;
  int32_t* out = idx + static_cast<int64_t>(t) * k;
  const int pos = tok_pos[t];
  if (pos < 0 || pos > max_pos) {
    if (c == 0) {
      if (threadIdx.x == 0) record_error(kErrBadIndex);
      for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = -1;
    }
    return;
  }
  const int n = pos + 1;
  if (n <= k) {
    if (c == 0)
      for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  const float* row = logits + static_cast<int64_t>(t) * ld;
  const int c0 = static_cast<int>(static_cast<int64_t>(n) * c / chunks);
  const int c1 = static_cast<int>(static_cast<int64_t>(n) * (c + 1) / chunks);
  // this CTA's chunk: asynchronous copies into shared memory, in flight while the
  // histogram is read and the threshold bucket chosen
  float* ck = reinterpret_cast<float*>(topk_smem_raw + kTopkSmemBase);
  for (int i = threadIdx.x; i < c1 - c0; i += blockDim.x) cp_async_4(ck + i, row + c0 + i);
  cp_async_commit();
  for (int b = threadIdx.x; b < 2048; b += blockDim.x)
    sm->hist[b] = ws.hist[static_cast<size_t>(t) * 2048 + b];
  __syncthreads();
  select_bucket(sm, 2048, k);
  const uint32_t b1 = static_cast<uint32_t>(sm->sel[0]);
  const int above1 = sm->sel[1];
  const int n_cand = sm->sel[2];
  cp_async_wait<0>();
  __syncthreads();
  int32_t* sa = ws.scr_a + static_cast<int64_t>(t) * ld;
  int2* sb = ws.scr_b + static_cast<int64_t>(t) * ld;
  struct ChunkKeys {
    const float* v;
    int off;
    __device__ uint32_t key(int i) const { return float_to_ordered(v[i]); }
    __device__ int index(int i) const { return off + i; }
  };
  const int2 cnt = ordered_pass_seg<kDecPerThread>(
      sm, ChunkKeys{ck, c0}, c1 - c0,
      [b1](uint32_t key) { return (key >> 21) > b1 ? 1 : ((key >> 21) == b1 ? 2 : 0); },
      [sa, c0](int r, uint32_t, int i) { sa[c0 + r] = i; },
      [sb, c0](int r, uint32_t key, int i) { sb[c0 + r] = make_int2(i, static_cast<int>(key)); },
      c1 - c0);
  if (threadIdx.x == 0) {
    ws.counts[(static_cast<size_t>(t) * chunks + c) * 2] = cnt.x;
    ws.counts[(static_cast<size_t>(t) * chunks + c) * 2 + 1] = cnt.y;
    __threadfence();
    const uint32_t prev = atomicAdd(&ws.arrive[t], 1u);
    sm->sel[3] = (prev == static_cast<uint32_t>(chunks - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!sm->sel[3]) return;
  __threadfence();
  // ---- the last CTA of this row finishes it; every step issues its global loads together.
  if (threadIdx.x < 32) {
    // prefix sums of the per-chunk counts (chunks <= kTopkMaxChunks = 4 x 32)
    const int lane = threadIdx.x;
    int carry_a = 0, carry_b = 0;
    for (int base = 0; base < chunks; base += 32) {
      const int cc = base + lane;
      const int va = cc < chunks ? ws.counts[(static_cast<size_t>(t) * chunks + cc) * 2] : 0;
      const int vb = cc < chunks ? ws.counts[(static_cast<size_t>(t) * chunks + cc) * 2 + 1] : 0;
      int ia = va, ib = vb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, ia, o), yb = __shfl_up_sync(0xffffffffu, ib, o);
        if (lane >= o) {
          ia += ya;
          ib += yb;
        }
      }
      if (cc < chunks) {
        sm->pre_a[cc + 1] = carry_a + ia;
        sm->pre_b[cc + 1] = carry_b + ib;
      }
      carry_a += __shfl_sync(0xffffffffu, ia, 31);
      carry_b += __shfl_sync(0xffffffffu, ib, 31);
    }
    if (lane == 0) {
      sm->pre_a[0] = 0;
      sm->pre_b[0] = 0;
    }
  }
  __syncthreads();
  // chunk holding flat entry g of a prefix array (largest cc with pre[cc] <= g)
  auto chunk_of = [&](const int* pre, int g) {
    int lo = 0, hi = chunks;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= g) lo = mid;
      else hi = mid;
    }
    return lo;
  };
  auto chunk_start = [&](int cc) { return static_cast<int>(static_cast<int64_t>(n) * cc / chunks); };
  const int got_a = sm->pre_a[chunks], got_b = sm->pre_b[chunks];
  const int k2 = k - got_a;
  // the counts actually gathered decide (they equal the histogram's when all is well)
  if (got_a != above1 || got_b != n_cand || k2 < 1 || k2 > got_b) {
    if (threadIdx.x == 0) record_error(kErrBadIndex);
    for (int i = threadIdx.x; i < k; i += blockDim.x) out[i] = -1;
    return;
  }
  // The finals (in chunk order) and the first batch of candidates: every load is issued
  // before any store, so the two gathers share one round trip.
  constexpr int kFin = (kMaxTopK + kTopkDecThreads - 1) / kTopkDecThreads;
  constexpr int kCandBatch = 4;
  const bool cand_in_smem = got_b <= kTopkCand;
  auto load_cands = [&](int g0, int2* cv) {
#pragma unroll
    for (int u = 0; u < kCandBatch; ++u) {
      const int g = g0 + u * kTopkDecThreads + threadIdx.x;
      cv[u] = make_int2(0, 0);
      if (g < got_b) {
        const int cc = chunk_of(sm->pre_b, g);
        cv[u] = sb[chunk_start(cc) + g - sm->pre_b[cc]];
      }
    }
  };
  auto store_cands = [&](int g0, const int2* cv) {
#pragma unroll
    for (int u = 0; u < kCandBatch; ++u) {
      const int g = g0 + u * kTopkDecThreads + threadIdx.x;
      if (g < got_b) {
        sm->cand_idx[g] = cv[u].x;
        sm->cand_key[g] = static_cast<uint32_t>(cv[u].y);
      }
    }
  };
  {
    int32_t v[kFin];
    int2 cv[kCandBatch];
#pragma unroll
    for (int u = 0; u < kFin; ++u) {
      const int g = u * kTopkDecThreads + threadIdx.x;
      v[u] = 0;
      if (g < got_a) {
        const int cc = chunk_of(sm->pre_a, g);
        v[u] = sa[chunk_start(cc) + g - sm->pre_a[cc]];
      }
    }
    if (cand_in_smem) load_cands(0, cv);
#pragma unroll
    for (int u = 0; u < kFin; ++u) {
      const int g = u * kTopkDecThreads + threadIdx.x;
      if (g < got_a) out[g] = v[u];
    }
    if (cand_in_smem) store_cands(0, cv);
  }
  if (cand_in_smem) {
    for (int g0 = kCandBatch * kTopkDecThreads; g0 < got_b; g0 += kCandBatch * kTopkDecThreads) {
      int2 cv[kCandBatch];
      load_cands(g0, cv);
      store_cands(g0, cv);
    }
    __syncthreads();
    finish_candidates(sm, RowCand{sm->cand_key, sm->cand_idx}, got_b, b1, k2, out + got_a);
  } else {
    // too many candidates for shared memory: compact them (position, key) into the front
    // of this row's candidate scratch (in place: entry g moves to g or lower) and resolve
    // from global memory
    for (int g0 = 0; g0 < got_b; g0 += blockDim.x) {  // same trip count in every thread
      const int g = g0 + threadIdx.x;
      int2 e = make_int2(0, 0);
      if (g < got_b) {
        const int cc = chunk_of(sm->pre_b, g);
        e = sb[chunk_start(cc) + g - sm->pre_b[cc]];
      }
      __syncthreads();
      if (g < got_b) sb[g] = e;
      __syncthreads();
    }
    __threadfence_block();
    __syncthreads();
    finish_candidates(sm, CandPairs{sb}, got_b, b1, k2, out + got_a);
  }
}

size_t topk_decode_ws_bytes(int32_t T, int64_t ld, int chunks) {
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  return al(static_cast<size_t>(T) * 2048 * 4) + al(static_cast<size_t>(T) * 4) +
         al(static_cast<size_t>(T) * chunks * 8) + al(static_cast<size_t>(T) * ld * 4) +
         al(static_cast<size_t>(T) * ld * 8);
}

// Largest chunk a CTA of the decode kernel reads (rows are at most max_pos + 1 long).
static size_t decode_chunk_cap(int32_t max_pos, int chunks) {
  return (static_cast<size_t>(max_pos) + 1 + chunks - 1) / chunks + 1;
}

int topk_decode_chunks(int32_t T, int32_t max_pos) {
  int c = T > 0 ? num_sms() / T : 1;
  // a chunk must fit the shared-memory row cache
  const int min_c = static_cast<int>((static_cast<size_t>(max_pos) + kTopkRowCache) / kTopkRowCache);
  if (c < min_c) c = min_c;
  const int by_len = (max_pos + 1) / 1024 + 1;
  if (c > by_len) c = by_len;
  if (c > kTopkMaxChunks) c = kTopkMaxChunks;
  return c < 1 ? 1 : c;
}

TopkDecodeLayout topk_decode_layout(void* ws, int32_t T, int64_t ld, int chunks) {
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  uint8_t* p = static_cast<uint8_t*>(ws);
  TopkDecodeLayout L;
  L.hist = reinterpret_cast<uint32_t*>(p);
  p += al(static_cast<size_t>(T) * 2048 * 4);
  L.arrive = reinterpret_cast<uint32_t*>(p);
  p += al(static_cast<size_t>(T) * 4);
  L.zero_words = (p - static_cast<uint8_t*>(ws)) / 4;
  L.counts = reinterpret_cast<int32_t*>(p);
  p += al(static_cast<size_t>(T) * chunks * 8);
  L.scr_a = reinterpret_cast<int32_t*>(p);
  p += al(static_cast<size_t>(T) * ld * 4);
  L.scr_b = reinterpret_cast<int2*>(p);
  return L;
}

cudaError_t launch_topk_decode(const float* logits, int64_t ld, const dsa_queries* q, int32_t k,
                               int32_t* idx, const TopkDecodeLayout& L, int chunks,
                               cudaStream_t stream) {
  if (q->n_tokens == 0) return cudaSuccess;
  static int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(topk_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kTopkSmemMax));
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  TopkDecodeWs w{L.hist, L.arrive, L.counts, L.scr_a, L.scr_b};
  const size_t cap = decode_chunk_cap(q->max_pos, chunks);
  if (cap > static_cast<size_t>(kTopkRowCache)) return cudaErrorNotSupported;
  const size_t smem = kTopkSmemBase + cap * sizeof(uint32_t);
  return launch_pdl(topk_decode_kernel, dim3(chunks, q->n_tokens), dim3(kTopkDecThreads), smem,
                    stream, logits, ld, q->tok_pos, q->max_pos, k, idx, w, chunks);
}

}  // namespace dsa
