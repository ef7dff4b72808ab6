// Cold pool -> HBM pool gather of the kept blocks, block-table construction, and the
// small per-pass / per-step kernels of the decode loop driver.
//
// Section 2, step 3 of "FlashMemory-DeepSeek-V4 Explained" (zhichai.net): the blocks
// the indexer keeps are moved from the CPU cold pool to the GPU before the next 64
// decode steps attend to them. The pool pages are read by the SMs straight from pinned
// host memory (mapped into the device address space) with 16-byte loads, eight in
// flight per thread, so the selected ids never travel back to the host.
#include "lsa_common.cuh"

namespace lsa {
namespace gth {

constexpr int THREADS = 256;
constexpr int MAX_B = 4096;          // sequences per call (prefix sums live in shared memory)
constexpr int UNROLL = 8;
constexpr int MAX_DELTA_GRID = 1024;  // CTAs of the delta gather (cooperative)

struct GatherArgs {
  const uint16_t* host_pool;
  long long host_blocks;
  const int64_t* host_blk_off;
  const int32_t* sel_ids;
  const int32_t* sel_cnt;
  const int32_t* res_pages;
  const int32_t* n_res;
  uint16_t* hbm_pool;
  long long n_pages;
  int32_t* block_table;
  int32_t* n_entries;
  int32_t* err;
  int cap, res_stride, B, d, sel_page_base, sel_page_count, bt_stride;
};

// Copy one [2][64][d] bf16 block (256*d bytes) with the whole CTA.
__device__ __forceinline__ void copy_block(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                           int n16) {
  for (int i0 = threadIdx.x; i0 < n16; i0 += THREADS * UNROLL) {
    uint4 v[UNROLL];
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
      const int i = i0 + k * THREADS;
      if (i < n16) v[k] = __ldcs(src + i);
    }
#pragma unroll
    for (int k = 0; k < UNROLL; ++k) {
      const int i = i0 + k * THREADS;
      if (i < n16) __stcs(dst + i, v[k]);
    }
  }
}

__global__ void __launch_bounds__(THREADS) gather_kernel(const GatherArgs a) {
  __shared__ int s_pref[MAX_B + 1];  // exclusive prefix of the kept-block counts
  __shared__ int s_warp[THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int carry = 0;
  for (int b0 = 0; b0 < a.B; b0 += THREADS) {
    const int b = b0 + tid;
    int c = 0;
    if (b < a.B) {
      c = __ldg(a.sel_cnt + b);
      c = c < 0 ? 0 : (c > a.cap ? a.cap : c);
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int before = carry;
    for (int k = 0; k < warp; ++k) before += s_warp[k];
    if (b < a.B) s_pref[b] = before + incl - c;
    int tot = 0;
    for (int k = 0; k < THREADS / 32; ++k) tot += s_warp[k];
    carry += tot;
    __syncthreads();
  }
  if (tid == 0) s_pref[a.B] = carry;
  __syncthreads();
  const int total = s_pref[a.B];

  // resident pages (window, tail last) after each sequence's kept blocks
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
    const int cnt = s_pref[b + 1] - s_pref[b];
    int nr = __ldg(a.n_res + b);
    if (nr < 0 || nr > a.res_stride || cnt + nr > a.bt_stride) {
      if (tid == 0) set_err(a.err, LSA_DEVERR_BAD_SIZE);
      nr = 0;
    }
    int32_t* bt = a.block_table + static_cast<long long>(b) * a.bt_stride;
    for (int i = tid; i < nr; i += THREADS)
      bt[cnt + i] = __ldg(a.res_pages + static_cast<long long>(b) * a.res_stride + i);
    if (tid == 0) a.n_entries[b] = cnt + nr;
  }

  // kept blocks: item k goes to page sel_page_base + k
  const int n16 = 16 * a.d;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    int lo = 0, hi = a.B - 1;  // last b with s_pref[b] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pref[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int b = lo, j = item - s_pref[b];
    const int c = __ldg(a.sel_ids + static_cast<long long>(b) * a.cap + j);
    const long long page = static_cast<long long>(a.sel_page_base) + item;
    const long long src = __ldg(a.host_blk_off + b) + c;
    const bool fits = item < a.sel_page_count && page < a.n_pages;
    const bool valid = c >= 0 && src >= 0 && src < a.host_blocks;
    if (tid == 0) {
      if (!fits) set_err(a.err, LSA_DEVERR_POOL_CAPACITY);
      if (!valid) set_err(a.err, LSA_DEVERR_BAD_PAGE);
      a.block_table[static_cast<long long>(b) * a.bt_stride + j] =
          (fits && valid) ? static_cast<int32_t>(page) : -1;
    }
    if (!fits || !valid) continue;
    copy_block(reinterpret_cast<const uint4*>(a.host_pool + src * 128 * a.d),
               reinterpret_cast<uint4*>(a.hbm_pool + page * 128 * a.d), n16);
  }
}

// ------------------------------------------------- delta gather (resident-page reuse)
// Section 2, step 5 ("refresh the loaded set"): a block kept in both the previous and the
// current pass keeps its HBM page; only the blocks new to this pass cross the host link,
// into pages that no kept block holds any more. One cooperative launch, four phases split
// by grid barriers:
//   0  clear the page bitmap;
//   1  each kept block is looked up (binary search) in its sequence's resident list of
//      the previous pass: a hit reuses that page (bit set in the bitmap), a miss is left
//      pending; each CTA counts its pending blocks;
//   2  each CTA counts the free pages of its share of the page range;
//   3  the k-th pending block (in sequence order) takes the k-th free page and is copied;
//      the resident lists become this pass's kept blocks and their pages.
struct DeltaArgs {
  GatherArgs g;
  int32_t* kept_ids;      // [B][cap] resident kept blocks (ascending ids), in and out
  int32_t* kept_pages;    // [B][cap] their pages
  int32_t* kept_cnt;      // [B]
  uint32_t* bitmap;       // [ceil(sel_page_count / 32)] pages held by a reused block
  int32_t* item_page;     // [B * cap] phase 1 decision per item (-1: pending)
  int32_t* cta_pend;      // [grid] pending blocks per CTA
  int32_t* cta_free;      // [grid] free pages per CTA share
  unsigned int* sync;     // [2] barrier arrivals, departures (left at zero)
  int32_t* copied;        // nullable [1]: blocks copied this call (accumulated)
};

__device__ __forceinline__ void delta_sync(const DeltaArgs& a, int* abort, unsigned int k) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(a.sync, 1u);
    const unsigned int target = k * gridDim.x;
    if (!*abort && !spin_until_geq(a.sync, target)) {
      set_err(a.g.err, LSA_DEVERR_TIMEOUT);
      *abort = 1;
    }
    __threadfence();
  }
  __syncthreads();
}

// Block-wide exclusive scan of one int per thread (THREADS threads); returns the total.
__device__ __forceinline__ int block_scan(int v, int& excl, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
  for (int k = 0; k < THREADS / 32; ++k) {
    if (k < warp) before += s_warp[k];
    total += s_warp[k];
  }
  __syncthreads();
  excl = before + incl - v;
  return total;
}

__global__ void __launch_bounds__(THREADS) gather_delta_kernel(const DeltaArgs d) {
  const GatherArgs& a = d.g;
  __shared__ int s_pref[MAX_B + 1];  // exclusive prefix of the kept-block counts
  __shared__ int s_warp[THREADS / 32];
  __shared__ int s_abort, s_base;
  __shared__ int s_fpre[MAX_DELTA_GRID + 1];   // free-page prefix over the CTAs' shares
  __shared__ int s_pend[MAX_DELTA_GRID];
  __shared__ int s_newpg[THREADS], s_item_b[THREADS], s_item_j[THREADS];
  const int tid = threadIdx.x;
  const int G = gridDim.x, cta = blockIdx.x;
  if (tid == 0) s_abort = 0;
  int carry = 0;
  for (int b0 = 0; b0 < a.B; b0 += THREADS) {
    const int b = b0 + tid;
    int c = 0;
    if (b < a.B) {
      c = __ldg(a.sel_cnt + b);
      c = c < 0 ? 0 : (c > a.cap ? a.cap : c);
    }
    int ex;
    const int tot = block_scan(c, ex, s_warp);
    if (b < a.B) s_pref[b] = carry + ex;
    carry += tot;
  }
  if (tid == 0) s_pref[a.B] = carry;
  __syncthreads();
  const int T = s_pref[a.B];
  const int PC = a.sel_page_count;
  const int nbw = (PC + 31) >> 5;
  // ---- phase 0: clear this CTA's share of the bitmap
  {
    const int w0 = static_cast<int>((static_cast<long long>(cta) * nbw) / G);
    const int w1 = static_cast<int>((static_cast<long long>(cta + 1) * nbw) / G);
    for (int w = w0 + tid; w < w1; w += THREADS) d.bitmap[w] = 0u;
  }
  delta_sync(d, &s_abort, 1);
  // ---- phase 1: reuse lookups; resident window pages after each sequence's kept blocks
  for (int b = cta; b < a.B; b += G) {
    const int cnt = s_pref[b + 1] - s_pref[b];
    int nr = __ldg(a.n_res + b);
    if (nr < 0 || nr > a.res_stride || cnt + nr > a.bt_stride) {
      if (tid == 0) set_err(a.err, LSA_DEVERR_BAD_SIZE);
      nr = 0;
    }
    int32_t* bt = a.block_table + static_cast<long long>(b) * a.bt_stride;
    for (int i = tid; i < nr; i += THREADS)
      bt[cnt + i] = __ldg(a.res_pages + static_cast<long long>(b) * a.res_stride + i);
    if (tid == 0) a.n_entries[b] = cnt + nr;
  }
  const int i0 = static_cast<int>((static_cast<long long>(cta) * T) / G);
  const int i1 = static_cast<int>((static_cast<long long>(cta + 1) * T) / G);
  int pend = 0;
  for (int item = i0 + tid; item < i1; item += THREADS) {
    int lo = 0, hi = a.B - 1;  // last b with s_pref[b] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pref[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int b = lo, j = item - s_pref[b];
    const int c = __ldg(a.sel_ids + static_cast<long long>(b) * a.cap + j);
    int kc = d.kept_cnt[b];
    kc = kc < 0 ? 0 : (kc > a.cap ? a.cap : kc);
    const int32_t* ki = d.kept_ids + static_cast<long long>(b) * a.cap;
    int l2 = 0, h2 = kc;                   // first position with id >= c
    while (l2 < h2) {
      const int mid = (l2 + h2) >> 1;
      if (ki[mid] < c) l2 = mid + 1; else h2 = mid;
    }
    int page = -1;
    if (l2 < kc && ki[l2] == c) {
      const int pg = d.kept_pages[static_cast<long long>(b) * a.cap + l2];
      const int rel = pg - a.sel_page_base;
      if (rel >= 0 && rel < PC) {
        page = pg;
        atomicOr(d.bitmap + (rel >> 5), 1u << (rel & 31));
      }
    }
    d.item_page[item] = page;
    if (page >= 0) a.block_table[static_cast<long long>(b) * a.bt_stride + j] = page;
    else ++pend;
  }
  {
    int ex;
    const int tot = block_scan(pend, ex, s_warp);
    if (tid == 0) d.cta_pend[cta] = tot;
  }
  delta_sync(d, &s_abort, 2);
  // ---- phase 2: free pages of this CTA's share of the page range
  const int p0 = static_cast<int>((static_cast<long long>(cta) * PC) / G);
  const int p1 = static_cast<int>((static_cast<long long>(cta + 1) * PC) / G);
  {
    int fr = 0;
    for (int pg = p0 + tid; pg < p1; pg += THREADS)
      fr += (__ldcg(d.bitmap + (pg >> 5)) >> (pg & 31)) & 1u ? 0 : 1;
    int ex;
    const int tot = block_scan(fr, ex, s_warp);
    if (tid == 0) d.cta_free[cta] = tot;
  }
  delta_sync(d, &s_abort, 3);
  // ---- phase 3: pending blocks take free pages in order and are copied
  if (!s_abort) {
    // free-page prefix over the CTAs' shares, and this CTA's pending-block offset
    for (int c = tid; c < G; c += THREADS) {
      s_fpre[c + 1] = __ldcg(d.cta_free + c);
      s_pend[c] = __ldcg(d.cta_pend + c);
    }
    __syncthreads();
    if (tid == 0) {
      s_fpre[0] = 0;
      for (int c = 0; c < G; ++c) s_fpre[c + 1] += s_fpre[c];
      int pre = 0;
      for (int c = 0; c < cta; ++c) pre += s_pend[c];
      s_base = pre;
    }
    __syncthreads();
    const int total_free = s_fpre[G];
    int rank_base = s_base;
    const int n16 = 16 * a.d;
    for (int base = i0; base < i1; base += THREADS) {
      const int item = base + tid;
      const bool mine = item < i1;
      const int pg0 = mine ? __ldcg(d.item_page + item) : 0;
      const int is_p = (mine && pg0 < 0) ? 1 : 0;
      int ex;
      const int tot = block_scan(is_p, ex, s_warp);
      int b = 0, j = 0, page = pg0;
      s_newpg[tid] = -1;
      if (mine) {
        int lo = 0, hi = a.B - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_pref[mid] <= item) lo = mid; else hi = mid - 1;
        }
        b = lo;
        j = item - s_pref[b];
        s_item_b[tid] = b;
        s_item_j[tid] = j;
      }
      if (is_p) {
        const int k = rank_base + ex;    // k-th pending block -> k-th free page
        page = -1;
        if (k < total_free) {
          int lo = 0, hi = G - 1;        // the share holding free page k
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_fpre[mid] <= k) lo = mid; else hi = mid - 1;
          }
          int want = k - s_fpre[lo];
          const int q0 = static_cast<int>((static_cast<long long>(lo) * PC) / G);
          const int q1 = static_cast<int>((static_cast<long long>(lo + 1) * PC) / G);
          for (int pg = q0; pg < q1; ++pg) {
            if (((__ldcg(d.bitmap + (pg >> 5)) >> (pg & 31)) & 1u) == 0) {
              if (want == 0) {
                page = a.sel_page_base + pg;
                break;
              }
              --want;
            }
          }
        } else {
          set_err(a.err, LSA_DEVERR_POOL_CAPACITY);
        }
        const int c = __ldg(a.sel_ids + static_cast<long long>(b) * a.cap + j);
        const long long src = __ldg(a.host_blk_off + b) + c;
        if (c < 0 || src < 0 || src >= a.host_blocks) {
          set_err(a.err, LSA_DEVERR_BAD_PAGE);
          page = -1;
        }
        a.block_table[static_cast<long long>(b) * a.bt_stride + j] = page;
        s_newpg[tid] = page;
      }
      if (mine) {
        d.kept_ids[static_cast<long long>(b) * a.cap + j] =
            __ldg(a.sel_ids + static_cast<long long>(b) * a.cap + j);
        d.kept_pages[static_cast<long long>(b) * a.cap + j] = page;
        if (j == s_pref[b + 1] - s_pref[b] - 1) d.kept_cnt[b] = j + 1;
      }
      rank_base += tot;
      __syncthreads();
      // this round's new blocks, each copied by the whole CTA
      const int nround = i1 - base < THREADS ? i1 - base : THREADS;
      for (int t = 0; t < nround; ++t) {
        const int pg = s_newpg[t];
        if (pg < 0) continue;
        const int bb = s_item_b[t], jj = s_item_j[t];
        const long long src = __ldg(a.host_blk_off + bb) +
                              __ldg(a.sel_ids + static_cast<long long>(bb) * a.cap + jj);
        copy_block(reinterpret_cast<const uint4*>(a.host_pool + src * 128 * a.d),
                   reinterpret_cast<uint4*>(a.hbm_pool + static_cast<long long>(pg) * 128 * a.d), n16);
        if (tid == 0 && d.copied != nullptr) atomicAdd(d.copied, 1);
      }
      __syncthreads();
    }
  }
  // sequences without kept blocks keep none
  for (int b = cta * THREADS + tid; b < a.B; b += G * THREADS)
    if (s_pref[b + 1] == s_pref[b]) d.kept_cnt[b] = 0;
  // ---- departure: the last CTA out resets the barrier counters
  __syncthreads();
  if (tid == 0) {
    if (atomicAdd(d.sync + 1, 1u) == static_cast<unsigned int>(G) - 1u) {
      atomicExch(d.sync, 0u);
      atomicExch(d.sync + 1, 0u);
    }
  }
}

// ----------------------------------------------------------- decode loop driver kernels
struct StepArgs {
  const int32_t* nb0;
  const int64_t* host_blk_off;   // [B+1]
  uint16_t* host_pool;
  long long host_blocks;
  uint16_t* hbm_pool;
  int32_t* n_cand;
  int32_t* res_pages;
  int32_t* n_res;
  int32_t* tail_len;
  int32_t* kept_cnt;             // nullable: resident kept blocks (delta gather)
  int32_t* err;
  int B, d, wb, max_cand;
};

// window ring page of block j of sequence b
__device__ __forceinline__ long long ring_page(const StepArgs& a, int b, long long j) {
  return static_cast<long long>(b) * (a.wb + 1) + j % (a.wb + 1);
}

// Pass p set-up (one CTA per sequence): candidate count, resident page list (window
// blocks oldest first, then the new tail page), and a zeroed tail page.
__global__ void __launch_bounds__(THREADS) pass_setup_kernel(const StepArgs a, int p) {
  const int b = blockIdx.x, tid = threadIdx.x;
  // the indexer launched next waits for this kernel's completion before it reads
  // anything; letting it launch now overlaps its CTAs' set-up with this small kernel
  grid_dependents_launch();
  const long long nb = static_cast<long long>(__ldg(a.nb0 + b)) + p;
  const long long first = nb - a.wb > 0 ? nb - a.wb : 0;
  if (tid == 0) {
    long long nc = nb - a.wb;
    if (nc < 0) nc = 0;
    if (nc > a.max_cand) {
      set_err(a.err, LSA_DEVERR_BAD_SIZE);
      nc = a.max_cand;
    }
    a.n_cand[b] = static_cast<int32_t>(nc);
    a.n_res[b] = static_cast<int32_t>(nb - first + 1);
    a.tail_len[b] = 0;
    if (p == 0 && a.kept_cnt != nullptr) a.kept_cnt[b] = 0;   // a run starts with none resident
  }
  for (long long i = tid; i < nb - first + 1; i += THREADS)
    a.res_pages[static_cast<long long>(b) * (a.wb + 1) + i] =
        static_cast<int32_t>(ring_page(a, b, first + i));
  // the previous pass's tail page is complete: write it back to the cold pool
  if (p > 0) {
    const long long hb = __ldg(a.host_blk_off + b) + nb - 1;
    if (hb < __ldg(a.host_blk_off + b + 1) && hb < a.host_blocks) {
      const uint4* src = reinterpret_cast<const uint4*>(a.hbm_pool + ring_page(a, b, nb - 1) * 128 * a.d);
      uint4* dst = reinterpret_cast<uint4*>(a.host_pool + hb * 128 * a.d);
      for (int i = tid; i < 16 * a.d; i += THREADS) dst[i] = src[i];
    } else if (tid == 0) {
      set_err(a.err, LSA_DEVERR_BAD_PAGE);
    }
    __syncthreads();  // with a one-page ring the new tail page is the old one
  }
  uint4* tail = reinterpret_cast<uint4*>(a.hbm_pool + ring_page(a, b, nb) * 128 * a.d);
  for (int i = tid; i < 16 * a.d; i += THREADS) tail[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Step s of pass p: write the new token's K and V into slot s of the tail page, write it
// through to the cold pool, and set tail_len = s + 1. One CTA per sequence, d/8 threads.
__global__ void append_kernel(const StepArgs a, int p, int s, const uint16_t* __restrict__ k_new,
                              const uint16_t* __restrict__ v_new) {
  const int b = blockIdx.x, t = threadIdx.x;
  const long long nb = static_cast<long long>(__ldg(a.nb0 + b)) + p;
  const long long page = ring_page(a, b, nb);
  const uint4 k = reinterpret_cast<const uint4*>(k_new + static_cast<long long>(b) * a.d)[t];
  const uint4 v = reinterpret_cast<const uint4*>(v_new + static_cast<long long>(b) * a.d)[t];
  reinterpret_cast<uint4*>(a.hbm_pool + (page * 128 + s) * a.d)[t] = k;
  reinterpret_cast<uint4*>(a.hbm_pool + (page * 128 + 64 + s) * a.d)[t] = v;
  const long long hb = __ldg(a.host_blk_off + b) + nb;
  if (hb < __ldg(a.host_blk_off + b + 1) && hb < a.host_blocks) {
    reinterpret_cast<uint4*>(a.host_pool + (hb * 128 + s) * a.d)[t] = k;
    reinterpret_cast<uint4*>(a.host_pool + (hb * 128 + 64 + s) * a.d)[t] = v;
  } else if (t == 0) {
    set_err(a.err, LSA_DEVERR_BAD_PAGE);
  }
  if (t == 0) a.tail_len[b] = s + 1;
}

// Load the window blocks of pass p from the cold pool into the rings. grid (wb, B).
__global__ void __launch_bounds__(THREADS) load_window_kernel(const StepArgs a, int p) {
  const int i = blockIdx.x, b = blockIdx.y;
  const long long nb = static_cast<long long>(__ldg(a.nb0 + b)) + p;
  const long long blk = nb - a.wb + i;
  if (blk < 0) return;
  const long long src = __ldg(a.host_blk_off + b) + blk;
  if (src >= __ldg(a.host_blk_off + b + 1) || src >= a.host_blocks) {
    if (threadIdx.x == 0) set_err(a.err, LSA_DEVERR_BAD_PAGE);
    return;
  }
  copy_block(reinterpret_cast<const uint4*>(a.host_pool + src * 128 * a.d),
             reinterpret_cast<uint4*>(a.hbm_pool + ring_page(a, b, blk) * 128 * a.d), 16 * a.d);
}

}  // namespace gth
}  // namespace lsa

// ------------------------------------------------------------------------ host side
namespace lsa_host {

// Device-visible address of pinned host memory (the same pointer under unified
// addressing); nullptr if `p` is not page-locked host memory.
const void* mapped_host_ptr(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) return nullptr;
  return at.devicePointer;
}

}  // namespace lsa_host

extern "C" lsa_status lsa_gather(const uint16_t* host_pool, int64_t host_blocks,
                                 const int64_t* host_blk_off, const int32_t* sel_ids,
                                 const int32_t* sel_cnt, int32_t cap, const int32_t* res_pages,
                                 const int32_t* n_res, int32_t res_stride, int32_t B, int32_t d,
                                 uint16_t* hbm_pool, int64_t n_pages, int32_t sel_page_base,
                                 int32_t sel_page_count, int32_t* block_table, int32_t bt_stride,
                                 int32_t* n_entries, int32_t* err, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_gather");
  if (!host_pool || !host_blk_off || !sel_cnt || !res_pages || !n_res || !hbm_pool ||
      !block_table || !n_entries || !err)
    return LSA_ERR_INVALID_ARG;
  if (cap > 0 && !sel_ids) return LSA_ERR_INVALID_ARG;
  if (B <= 0 || B > lsa::gth::MAX_B || d <= 0 || d % 8 != 0 || cap < 0 || res_stride < 0 ||
      host_blocks <= 0 || n_pages <= 0 || sel_page_base < 0 || sel_page_count < 0 ||
      bt_stride < cap + res_stride)
    return LSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(sel_page_base) + sel_page_count > n_pages) return LSA_ERR_INVALID_ARG;
  const void* hp = lsa_host::mapped_host_ptr(host_pool);
  if (hp == nullptr) return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hp) | reinterpret_cast<uintptr_t>(hbm_pool)) & 15u)
    return LSA_ERR_INVALID_ARG;
  lsa::gth::GatherArgs a;
  a.host_pool = static_cast<const uint16_t*>(hp);
  a.host_blocks = host_blocks;
  a.host_blk_off = host_blk_off;
  a.sel_ids = sel_ids;
  a.sel_cnt = sel_cnt;
  a.res_pages = res_pages;
  a.n_res = n_res;
  a.hbm_pool = hbm_pool;
  a.n_pages = n_pages;
  a.block_table = block_table;
  a.n_entries = n_entries;
  a.err = err;
  a.cap = cap;
  a.res_stride = res_stride;
  a.B = B;
  a.d = d;
  a.sel_page_base = sel_page_base;
  a.sel_page_count = sel_page_count;
  a.bt_stride = bt_stride;
  const int G = lsa_host::sm_count();
  if (G <= 0) return LSA_ERR_CUDA;
  lsa::gth::gather_kernel<<<2 * G, lsa::gth::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

namespace {
inline size_t r256(size_t x) { return (x + 255) / 256 * 256; }
struct DeltaWs {
  size_t bitmap, item_page, cta_pend, cta_free, total;
};
DeltaWs delta_ws_layout(int B, int cap, int sel_page_count, int grid) {
  DeltaWs w;
  w.bitmap = 256;                                   // [0, 256): barrier counters
  w.item_page = w.bitmap + r256(static_cast<size_t>((sel_page_count + 31) / 32) * 4);
  w.cta_pend = w.item_page + r256(static_cast<size_t>(B) * (cap > 0 ? cap : 1) * 4);
  w.cta_free = w.cta_pend + r256(static_cast<size_t>(grid) * 4);
  w.total = w.cta_free + r256(static_cast<size_t>(grid) * 4);
  return w;
}
int delta_grid() {
  const int n = lsa_host::sm_count();
  const int g = 2 * n;
  return g < lsa::gth::MAX_DELTA_GRID ? g : lsa::gth::MAX_DELTA_GRID;
}
}  // namespace

extern "C" size_t lsa_gather_delta_workspace_size(int32_t B, int32_t cap, int32_t sel_page_count,
                                                  int32_t n_sm) {
  if (B <= 0 || cap < 0 || sel_page_count < 0 || n_sm <= 0) return 0;
  const int g = 2 * n_sm < lsa::gth::MAX_DELTA_GRID ? 2 * n_sm : lsa::gth::MAX_DELTA_GRID;
  return delta_ws_layout(B, cap, sel_page_count, g).total;
}

extern "C" lsa_status lsa_gather_delta(
    const uint16_t* host_pool, int64_t host_blocks, const int64_t* host_blk_off,
    const int32_t* sel_ids, const int32_t* sel_cnt, int32_t cap, const int32_t* res_pages,
    const int32_t* n_res, int32_t res_stride, int32_t B, int32_t d, uint16_t* hbm_pool,
    int64_t n_pages, int32_t sel_page_base, int32_t sel_page_count, int32_t* block_table,
    int32_t bt_stride, int32_t* n_entries, int32_t* kept_ids, int32_t* kept_pages,
    int32_t* kept_cnt, void* ws, size_t ws_bytes, int32_t* copied, int32_t* err, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_gather_delta");
  if (!host_pool || !host_blk_off || !sel_cnt || !res_pages || !n_res || !hbm_pool ||
      !block_table || !n_entries || !err || !kept_cnt || !ws)
    return LSA_ERR_INVALID_ARG;
  if (cap > 0 && (!sel_ids || !kept_ids || !kept_pages)) return LSA_ERR_INVALID_ARG;
  if (B <= 0 || B > lsa::gth::MAX_B || d <= 0 || d % 8 != 0 || cap < 0 || res_stride < 0 ||
      host_blocks <= 0 || n_pages <= 0 || sel_page_base < 0 || sel_page_count < 0 ||
      bt_stride < cap + res_stride)
    return LSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(sel_page_base) + sel_page_count > n_pages) return LSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 15u) return LSA_ERR_INVALID_ARG;
  const int G = delta_grid();
  if (G <= 0) return LSA_ERR_CUDA;
  const DeltaWs lay = delta_ws_layout(B, cap, sel_page_count, G);
  if (ws_bytes < lay.total) return LSA_ERR_INVALID_ARG;
  const void* hp = lsa_host::mapped_host_ptr(host_pool);
  if (hp == nullptr) return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(hp) | reinterpret_cast<uintptr_t>(hbm_pool)) & 15u)
    return LSA_ERR_INVALID_ARG;
  lsa::gth::DeltaArgs a;
  a.g.host_pool = static_cast<const uint16_t*>(hp);
  a.g.host_blocks = host_blocks;
  a.g.host_blk_off = host_blk_off;
  a.g.sel_ids = sel_ids;
  a.g.sel_cnt = sel_cnt;
  a.g.res_pages = res_pages;
  a.g.n_res = n_res;
  a.g.hbm_pool = hbm_pool;
  a.g.n_pages = n_pages;
  a.g.block_table = block_table;
  a.g.n_entries = n_entries;
  a.g.err = err;
  a.g.cap = cap;
  a.g.res_stride = res_stride;
  a.g.B = B;
  a.g.d = d;
  a.g.sel_page_base = sel_page_base;
  a.g.sel_page_count = sel_page_count;
  a.g.bt_stride = bt_stride;
  uint8_t* base = static_cast<uint8_t*>(ws);
  a.kept_ids = kept_ids;
  a.kept_pages = kept_pages;
  a.kept_cnt = kept_cnt;
  a.sync = reinterpret_cast<unsigned int*>(base);
  a.bitmap = reinterpret_cast<uint32_t*>(base + lay.bitmap);
  a.item_page = reinterpret_cast<int32_t*>(base + lay.item_page);
  a.cta_pend = reinterpret_cast<int32_t*>(base + lay.cta_pend);
  a.cta_free = reinterpret_cast<int32_t*>(base + lay.cta_free);
  a.copied = copied;
  // cooperative: the grid barriers need every CTA resident
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(lsa::gth::THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, lsa::gth::gather_delta_kernel, a) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

// ------------------------------------------------------------------ decode loop driver
namespace {
lsa::gth::StepArgs step_args(const lsa_state* st, const void* host_dev) {
  lsa::gth::StepArgs a;
  a.nb0 = st->nb0;
  a.host_blk_off = st->host_blk_off;
  a.host_pool = static_cast<uint16_t*>(const_cast<void*>(host_dev));
  a.host_blocks = st->host_blocks;
  a.hbm_pool = st->hbm_pool;
  a.n_cand = st->n_cand;
  a.res_pages = st->res_pages;
  a.n_res = st->n_res;
  a.tail_len = st->tail_len;
  a.kept_cnt = st->kept_cnt;
  a.err = st->err;
  a.B = st->B;
  a.d = st->d;
  a.wb = st->W / LSA_BLOCK;
  a.max_cand = st->max_cand;
  return a;
}
}  // namespace

extern "C" lsa_status lsa_load_window(const lsa_state* st, int32_t pass, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_load_window");
  const lsa_status v = lsa_state_check(st);
  if (v != LSA_OK) return v;
  if (pass < 0) return LSA_ERR_INVALID_ARG;
  const void* hp = lsa_host::mapped_host_ptr(st->host_pool);
  if (hp == nullptr) return LSA_ERR_INVALID_ARG;
  const lsa::gth::StepArgs a = step_args(st, hp);
  if (a.wb == 0) return LSA_OK;
  lsa::gth::load_window_kernel<<<dim3(a.wb, st->B), lsa::gth::THREADS, 0,
                                 static_cast<cudaStream_t>(stream)>>>(a, pass);
  return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

extern "C" lsa_status lsa_pass_setup(const lsa_state* st, int32_t pass, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_pass_setup");
  const lsa_status v = lsa_state_check(st);
  if (v != LSA_OK) return v;
  if (pass < 0) return LSA_ERR_INVALID_ARG;
  const void* hp = lsa_host::mapped_host_ptr(st->host_pool);
  if (hp == nullptr) return LSA_ERR_INVALID_ARG;
  lsa::gth::pass_setup_kernel<<<st->B, lsa::gth::THREADS, 0, static_cast<cudaStream_t>(stream)>>>(
      step_args(st, hp), pass);
  return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

extern "C" lsa_status lsa_append(const lsa_state* st, int64_t step, const uint16_t* k_new,
                                 const uint16_t* v_new, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_append");
  const lsa_status v = lsa_state_check(st);
  if (v != LSA_OK) return v;
  if (step < 0 || step / LSA_TAU > (int64_t(1) << 30) || !k_new || !v_new)
    return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15u)
    return LSA_ERR_INVALID_ARG;
  const void* hp = lsa_host::mapped_host_ptr(st->host_pool);
  if (hp == nullptr) return LSA_ERR_INVALID_ARG;
  lsa::gth::append_kernel<<<st->B, st->d / 8, 0, static_cast<cudaStream_t>(stream)>>>(
      step_args(st, hp), static_cast<int>(step / LSA_TAU), static_cast<int>(step % LSA_TAU),
      k_new, v_new);
  return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

extern "C" lsa_status lsa_decode_step(const lsa_state* st, int64_t step, const uint16_t* q,
                                      const uint16_t* k_new, const uint16_t* v_new, uint16_t* out,
                                      void* stream) {
  const lsa_status v = lsa_state_check(st);
  if (v != LSA_OK) return v;
  if (step < 0 || step / LSA_TAU > (int64_t(1) << 30) || !q || !k_new || !v_new || !out)
    return LSA_ERR_INVALID_ARG;
  lsa_host::AppendArgs ap;
  ap.k_new = k_new;
  ap.v_new = v_new;
  ap.tail_len_out = st->tail_len;
  ap.tail = static_cast<int>(step % LSA_TAU) + 1;
  return lsa_host::decode_attn(q, st->hbm_pool, st->n_pages, st->block_table, st->bt_stride,
                               st->n_entries, st->tail_len, st->B, st->H, st->d, st->scale, out,
                               st->attn_ws, st->attn_ws_bytes, st->err, stream, &ap);
}

extern "C" lsa_status lsa_step(const lsa_state* st, int64_t step, const uint16_t* h,
                               const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                               uint16_t* out, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_step");
  lsa_status v = lsa_state_check(st);
  if (v != LSA_OK) return v;
  if (step < 0 || step / LSA_TAU > (int64_t(1) << 30) || !q || !k_new || !v_new || !out)
    return LSA_ERR_INVALID_ARG;
  const int p = static_cast<int>(step / LSA_TAU), s = static_cast<int>(step % LSA_TAU);
  if (s == 0) {
    if (!h) return LSA_ERR_INVALID_ARG;
    v = lsa_pass_setup(st, p, stream);
    if (v != LSA_OK) return v;
    v = lsa_index_ex(h, st->w_q, st->bias, st->k_idx, st->kidx_layer_stride, st->kidx_off,
                     st->n_cand, st->B, st->L, st->D, st->d_i, st->max_cand, st->sel_ids,
                     st->sel_cnt, st->cap, nullptr, nullptr, st->index_ws, st->index_ws_bytes,
                     st->err, stream);
    if (v != LSA_OK) return v;
    const int wb1 = st->W / LSA_BLOCK + 1;
    const int64_t base = static_cast<int64_t>(st->B) * wb1;
    if (st->kept_cnt != nullptr)
      v = lsa_gather_delta(st->host_pool, st->host_blocks, st->host_blk_off, st->sel_ids,
                           st->sel_cnt, st->cap, st->res_pages, st->n_res, wb1, st->B, st->d,
                           st->hbm_pool, st->n_pages, static_cast<int32_t>(base),
                           static_cast<int32_t>(st->n_pages - base), st->block_table,
                           st->bt_stride, st->n_entries, st->kept_ids, st->kept_pages,
                           st->kept_cnt, st->gather_ws, st->gather_ws_bytes, nullptr, st->err,
                           stream);
    else
      v = lsa_gather(st->host_pool, st->host_blocks, st->host_blk_off, st->sel_ids, st->sel_cnt,
                     st->cap, st->res_pages, st->n_res, wb1, st->B, st->d, st->hbm_pool,
                     st->n_pages, static_cast<int32_t>(base),
                     static_cast<int32_t>(st->n_pages - base), st->block_table, st->bt_stride,
                     st->n_entries, st->err, stream);
    if (v != LSA_OK) return v;
  }
  return lsa_decode_step(st, step, q, k_new, v_new, out, stream);
}
