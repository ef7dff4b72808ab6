// Block-sparse split-K flash-decode MQA attention on the sm_100a tensor cores, and the
// log-sum-exp merge of its partial results.
//
// One decode step of section 2, step 4 of "FlashMemory-DeepSeek-V4 Explained"
// (zhichai.net): the query heads of a sequence attend only to the KV pages listed in its
// block table (the kept blocks, the recent window, the tail page of new tokens).
//
// Work split. A sequence's tokens are cut into 32-token units (a page is two units; the
// tail page ceil(tail_len/32)). All units of the batch, in sequence order, are divided
// evenly over the grid (one CTA per SM), so a CTA may finish one sequence and start the
// next; each (CTA, sequence) piece is a "segment" that leaves one partial result
// (unnormalised O, running max m, sum l) in the workspace slot CTA + sequence. Within a
// segment, tiles of 128 tokens (4 units) are processed in a software pipeline:
//
//   warp 0  TMA producer: Q once per segment, then K and V of each tile, in 16 KB
//           stages of [128 tokens][64 dims] (128-byte swizzle) through an 8-stage ring;
//   warp 1  MMA issuer (one thread): S^T[tok][head] = K . Q^T into tensor memory
//           (M = 128 tokens, N = heads, K = d), then O^T[dim][head] += V^T . P^T
//           (M = 128 dims per MMA, N = heads, K = 128 tokens), accumulated in TMEM;
//   warps 2-5 softmax: each owns 32 rows (tokens) of S^T, finds the per-head tile max
//           (warp butterfly + shared memory), keeps a running max per head that is only
//           raised when the tile max exceeds it by more than 2^8 (O^T in TMEM is then
//           rescaled), writes P^T = exp2(S*scale*log2e - m) as bf16 into shared memory,
//           and accumulates the per-head denominators in registers.
//
// Tensor memory columns: S^T double buffer [0, 2*HP), O^T blocks [2*HP, 2*HP + HP*d/128).
#include "lsa_common.cuh"

#include <math.h>

#include <atomic>
#include <mutex>

namespace lsa {
namespace attn {

constexpr int TILE = 128;                 // tokens per tile (the MMA M of S^T)
constexpr int UNIT = 32;                  // tokens per work unit (rows per TMA box)
constexpr int NST = 8;                    // stages in the K/V ring (even: V pairs stay adjacent)
constexpr int STAGE_BYTES = TILE * 128;   // [128 rows][64 bf16] = 16 KB
constexpr int NTHREADS = 192;
constexpr int MAXSEG = 16;                // segments planned per batch
constexpr float RESCALE_LOG2 = 8.0f;      // raise the running max only by more than 2^8
constexpr int MAXITEMS = 64;              // sequences a CTA's merge range meets, per round
constexpr int MAXRUNS = 64;               // (sequence, head, chunk range) runs per merge group
constexpr int SCRATCH_FLOATS = 4 * NTHREADS;  // merge scratch after a group's rows
constexpr int MAX_GRID = 256;             // CTAs per launch (one per SM)

struct Seg {
  int b, u0, u1;
};

struct Misc {
  uint64_t full[NST], empty[NST];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done, q_full, q_free, mma_done;
  uint64_t merge_bar;               // the merge's bulk copies of partial rows
  uint32_t tmem_base;
  int abort;
  int nseg, more;
  Seg seg[MAXSEG];
  float red[4][64];
  float m_use[64];
  float alpha[64];
  int resc_tile;                    // the last softmax tile in which some head rescaled
  // fused merge
  int n_items, total_items;
  long long merge_j0, merge_j1, cur_j;
  int cur_rec, n_runs, group_floats, precut;
  long long group_bytes;
  int item_b[MAXITEMS], item_h[MAXITEMS], item_clo[MAXITEMS], item_chi[MAXITEMS];
  int run_b[MAXRUNS], run_h[MAXRUNS], run_c0[MAXRUNS], run_nch[MAXRUNS], run_clo[MAXRUNS],
      run_n[MAXRUNS], run_off[MAXRUNS];
  float run_inv[MAXRUNS];
  long long ustart[MAX_GRID + 1];   // first unit of each CTA: floor(c * U / G)
};

struct Args {
  const int32_t* block_table;
  const int32_t* n_entries;
  const int32_t* tail_len;
  float* part_o;          // [d/128][H][slots][128] fp32: the rows a merge item needs (one
                          //   128-dim chunk of one head over consecutive slots) are contiguous
  float* part_ml;         // [H][slots][4] fp32 (running max in log2 units, denominator, two
                          //   pad words: 16 bytes, so a run's pairs come by one bulk copy)
  unsigned int* sync;     // [2] grid-barrier arrive / depart counters (left at zero)
  uint16_t* out;          // [B][H][d] bf16
  uint16_t* pool;         // the HBM pool (written only by the fused append)
  const uint16_t* k_new;  // fused append: [B][d] token written into slot fused_tail-1
  const uint16_t* v_new;  //   of each tail page (nullptr: no append)
  int32_t* tail_len_out;  // fused append: receives fused_tail per sequence (nullable)
  int32_t* err;
  long long n_pages;
  int bt_stride, B, H, d;
  int fused_tail;         // > 0: every sequence's tail length (tail_len is not read)
  float scale_log2;
};

// Units (32-token pieces) of sequence b; 0 for an empty or malformed sequence.
__device__ __forceinline__ int seq_tail(const Args& a, int b) {
  return a.fused_tail > 0 ? a.fused_tail : __ldg(a.tail_len + b);
}

__device__ __forceinline__ int seq_units(const Args& a, int b) {
  const int n = __ldg(a.n_entries + b);
  const int t = seq_tail(a, b);
  if (n <= 0 || n > a.bt_stride || t < 1 || t > 64) return 0;
  return 2 * (n - 1) + (t + UNIT - 1) / UNIT;
}

__device__ __forceinline__ bool seq_malformed(const Args& a, int b) {
  const int n = __ldg(a.n_entries + b);
  const int t = seq_tail(a, b);
  if (n < 0) return true;
  if (n == 0) return false;
  return n > a.bt_stride || t < 1 || t > 64;
}

// Total units of the batch, summed by one warp (all lanes get the result).
__device__ __forceinline__ long long warp_total_units(const Args& a, int lane) {
  long long s = 0;
  for (int b = lane; b < a.B; b += 32) s += seq_units(a, b);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// Warp 0: list the segments of units [us, ue), skipping the first `skip` of them; at most
// MAXSEG are stored. Sets m->more when segments remain after the stored ones.
__device__ __noinline__ void plan_segments(const Args& a, long long us, long long ue, int skip, Misc* m,
                              int lane) {
  int found = 0, stored = 0;
  bool more = false;
  long long base = 0;
  for (int b0 = 0; b0 < a.B && base < ue && !more; b0 += 32) {
    const int b = b0 + lane;
    const int u = b < a.B ? seq_units(a, b) : 0;
    long long incl = u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const long long p = base + incl - u;  // first unit of sequence b
    const bool hit = u > 0 && us < ue && p < ue && p + u > us;
    const unsigned mask = __ballot_sync(0xffffffffu, hit);
    if (hit) {
      const int idx = found + __popc(mask & ((1u << lane) - 1u)) - skip;
      if (idx >= MAXSEG) {
        more = true;
      } else if (idx >= 0) {
        Seg s;
        s.b = b;
        s.u0 = static_cast<int>(us > p ? us - p : 0);
        s.u1 = static_cast<int>((ue < p + u ? ue : p + u) - p);
        m->seg[idx] = s;
      }
    }
    more = __any_sync(0xffffffffu, more);
    found += __popc(mask);
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  stored = found - skip;
  if (stored < 0) stored = 0;
  if (stored > MAXSEG) stored = MAXSEG;
  if (lane == 0) {
    m->nseg = stored;
    m->more = (found - skip > MAXSEG) ? 1 : 0;
  }
}

// Units [tu0, tu1) of tile t of a segment. The segment's partial tile (fewer than 4
// units) comes first: its small loads overlap the pipeline fill, and the segment ends on
// full tiles, so a CTA with one unit more than another does not pay an extra round trip
// at the end.
__device__ __forceinline__ void tile_range(const Seg& sg, int t, int& tu0, int& tu1) {
  const int len = sg.u1 - sg.u0;
  const int first = (len & 3) ? (len & 3) : 4;
  if (t == 0) {
    tu0 = sg.u0;
    tu1 = sg.u0 + (first < len ? first : len);
  } else {
    tu0 = sg.u0 + first + 4 * (t - 1);
    tu1 = tu0 + 4 < sg.u1 ? tu0 + 4 : sg.u1;
  }
}

// Butterfly reduce-scatter over the 32 lanes of a warp: afterwards lane l holds the
// reduction of heads [l*N/32, l*N/32 + N/32) in v[0..] (N >= 32), or of head l/2 (N == 16).
template <int N, bool IS_MAX>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N], int lane) {
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
    if (n > 1) {
      const int half = n >> 1;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < half) {
          const float send = up ? v[i] : v[i + half];
          const float keep = up ? v[i + half] : v[i];
          const float recv = __shfl_xor_sync(0xffffffffu, send, o);
          v[i] = IS_MAX ? fmaxf(keep, recv) : keep + recv;
        }
      }
      n = half;
    } else {
      const float recv = __shfl_xor_sync(0xffffffffu, v[0], o);
      v[0] = IS_MAX ? fmaxf(v[0], recv) : v[0] + recv;
    }
  }
}

template <int N>
__device__ __forceinline__ void store_scattered(float* dst, const float (&v)[N], int lane) {
  if constexpr (N >= 32) {
#pragma unroll
    for (int i = 0; i < N / 32; ++i) dst[lane * (N / 32) + i] = v[i];
  } else {
    if ((lane & 1) == 0) dst[lane >> 1] = v[0];
  }
}

// 2^x on the special-function unit (relative error about 2^-22, results below 2^-126
// flushed to zero): the softmax weights are rounded to bf16 right after, so the extra
// care of exp2f for subnormal results buys nothing.
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// TMEM load of HP consecutive columns of this warp's 32 lanes.
template <int HP>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[HP]) {
#pragma unroll
  for (int c = 0; c < HP / 16; ++c) tmem_ld16(taddr + 16 * c, v + 16 * c);
}

// CTA holding unit u of the grid-wide split: the largest c with floor(c*U/G) <= u.
__device__ __forceinline__ long long cta_of_unit(long long u, long long U, long long G) {
  return ((u + 1) * G - 1) / U;
}
__device__ __forceinline__ bool cta_empty(long long c, long long U, long long G) {
  return (c * U) / G == ((c + 1) * U) / G;
}

// Merge work items are (sequence, head, 128-dim chunk) triples of every sequence whose
// units span more than one CTA (they are merged from partials) or that has no units at
// all (its output is zero-filled), numbered in sequence order. CTA c owns the
// contiguous item range [c*T/G, (c+1)*T/G), so a CTA's items mostly share a head.
//
// Warp 0: record the sequences that meet this CTA's item range, skipping the first
// `skip` of them (at most MAXITEMS are recorded). Also reports malformed sequences
// (each from one CTA only).
__device__ __noinline__ void plan_merge(const Args& a, long long U, int skip, Misc* m, int lane) {
  const long long G = gridDim.x;
  const int cta = blockIdx.x;
  const int n_chunks = a.d / 128;
  // pass 1: total items T
  long long T = 0;
  {
    long long base_u = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      const int u = b < a.B ? seq_units(a, b) : 0;
      if (b < a.B && b % G == cta && seq_malformed(a, b)) set_err(a.err, LSA_DEVERR_BAD_SIZE);
      long long incl = u;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const long long p = base_u + incl - u;
      bool has = false;
      if (b < a.B) has = (u == 0) || (cta_of_unit(p, U, G) != cta_of_unit(p + u - 1, U, G));
      long long items = has ? static_cast<long long>(a.H) * n_chunks : 0;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) items += __shfl_xor_sync(0xffffffffu, items, o);
      T += items;
      base_u += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  const long long j0 = (static_cast<long long>(cta) * T) / G;
  const long long j1 = (static_cast<long long>(cta + 1) * T) / G;
  // pass 2: sequences meeting [j0, j1)
  long long base_u = 0, base_i = 0;
  int found = 0;
  for (int b0 = 0; b0 < a.B && base_i < j1; b0 += 32) {
    const int b = b0 + lane;
    const int u = b < a.B ? seq_units(a, b) : 0;
    long long incl = u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const long long p = base_u + incl - u;
    long long clo = 0, chi = -1;
    bool has = false;
    if (b < a.B) {
      if (u == 0) {
        has = true;
      } else {
        clo = cta_of_unit(p, U, G);
        chi = cta_of_unit(p + u - 1, U, G);
        has = clo != chi;
      }
    }
    const long long items = has ? static_cast<long long>(a.H) * n_chunks : 0;
    long long iincl = items;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, iincl, o);
      if (lane >= o) iincl += t;
    }
    const long long ib = base_i + iincl - items;
    const bool hit = items > 0 && ib < j1 && ib + items > j0;
    const unsigned mask = __ballot_sync(0xffffffffu, hit);
    if (hit) {
      const int idx = found + __popc(mask & ((1u << lane) - 1u)) - skip;
      if (idx >= 0 && idx < MAXITEMS) {
        m->item_b[idx] = b;
        m->item_h[idx] = static_cast<int>(ib);  // first item of the sequence
        m->item_clo[idx] = static_cast<int>(clo);
        m->item_chi[idx] = static_cast<int>(chi);
      }
    }
    found += __popc(mask);
    base_u += __shfl_sync(0xffffffffu, incl, 31);
    base_i += __shfl_sync(0xffffffffu, iincl, 31);
  }
  if (lane == 0) {
    const int left = found - skip;
    m->n_items = left < 0 ? 0 : (left > MAXITEMS ? MAXITEMS : left);
    m->total_items = static_cast<int>(T > 0x7fffffff ? 0x7fffffff : T);
    m->merge_j0 = j0;
    m->merge_j1 = j1;
  }
}

// Block-wide reductions over the CTA's threads through m->red[0][*].
__device__ __forceinline__ float block_max(float v, Misc* m, int tid, int nwarps) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((tid & 31) == 0) m->red[0][tid >> 5] = v;
  __syncthreads();
  float r = m->red[0][0];
  for (int w = 1; w < nwarps; ++w) r = fmaxf(r, m->red[0][w]);
  return r;
}
__device__ __forceinline__ float block_sum(float v, Misc* m, int tid, int nwarps) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((tid & 31) == 0) m->red[0][tid >> 5] = v;
  __syncthreads();
  float r = 0.f;
  for (int w = 0; w < nwarps; ++w) r += m->red[0][w];
  return r;
}

constexpr int CW = 128;                   // merge chunk: head dimensions per partial row

// One thread: cut the next group of merge runs (one sequence, one head, a range of
// 128-dim chunks) from the CTA's recorded items, as many as fit `buf_floats` minus the
// output scratch. A run's region holds its nch chunks of n rows of CW floats, then n
// (m, l) pairs, then n weights (16-byte multiples, so that every chunk starts on a
// 16-byte boundary as bulk copies require). Sets n_runs, group_floats, group_bytes (the
// bytes the group's bulk copies bring) and advances cur_rec / cur_j.
__device__ __noinline__ void cut_group(const Args& a, Misc* m, int buf_floats) {
  const int nrec = m->n_items;
  const int nch_all = a.d / CW;
  int r = m->cur_rec, nr = 0;
  long long j = m->cur_j;
  long long used = 0, bytes = 0;
  while (r < nrec && nr < MAXRUNS) {
    const long long ib = m->item_h[r];
    const long long lo = m->merge_j0 > ib ? m->merge_j0 : ib;
    const long long hi_all = ib + static_cast<long long>(a.H) * nch_all;
    const long long hi = m->merge_j1 < hi_all ? m->merge_j1 : hi_all;
    if (j < lo) j = lo;
    if (j >= hi) {
      ++r;
      j = -1;
      continue;
    }
    const int rel = static_cast<int>(j - ib);   // < H * nch_all: 32-bit division
    const int h = rel / nch_all;
    const int c0 = rel - h * nch_all;
    long long run_end = ib + static_cast<long long>(h + 1) * nch_all;
    if (run_end > hi) run_end = hi;
    int nch = static_cast<int>(run_end - j);
    const int n = m->item_chi[r] - m->item_clo[r] + 1;   // 0: empty sequence
    const long long tail = 4LL * n + ((n + 3) & ~3LL);   // (m, l, pad, pad) and weights
    long long need = static_cast<long long>(nch) * n * CW + tail;
    if (used + need > buf_floats - SCRATCH_FLOATS) {
      if (nr > 0) break;
      nch = static_cast<int>((buf_floats - SCRATCH_FLOATS - tail) / (n > 0 ? static_cast<long long>(CW) * n : 1));
      if (nch < 1) nch = 1;     // n <= MAX_GRID: one chunk (128 KB) always fits
      need = static_cast<long long>(nch) * n * CW + tail;
    }
    m->run_b[nr] = m->item_b[r];
    m->run_h[nr] = h;
    m->run_c0[nr] = c0;
    m->run_nch[nr] = nch;
    m->run_clo[nr] = m->item_clo[r];
    m->run_n[nr] = n;
    m->run_off[nr] = static_cast<int>(used);
    used += need;
    bytes += static_cast<long long>(nch) * n * CW * 4 + 16LL * n;
    j += nch;
    ++nr;
  }
  m->cur_rec = r;
  m->cur_j = j;
  m->n_runs = nr;
  m->group_floats = static_cast<int>(used);
  m->group_bytes = bytes;
}

// Fused log-sum-exp merge, run by every thread of every CTA after its segments:
//   M = max_k m_k,  out = sum_k 2^(m_k - M) O_k / sum_k 2^(m_k - M) l_k   (m in log2 units)
// over the partials k of a split sequence. A grid-wide barrier (one arrival counter,
// bounded wait) separates the partial writes from the reads. The CTA's items are cut
// into runs (one sequence, one head, a range of 128-dim chunks; the first group is cut
// before the barrier). In the partial layout the rows of one chunk of one head over
// consecutive slots are contiguous, so a run needs one 1-D bulk copy per chunk and one
// for its (m, l) pairs; all the group's copies are issued at once (spread over the
// threads): one round trip per group. One warp per run derives the split weights from
// shared memory; then the threads of a warp take consecutive 16-byte
// columns of one run and walk the same split rows, each slice of the threads a
// contiguous range of the splits, and the slices meet in scratch.
__device__ __forceinline__ void merge_phase(const Args& a, Misc* m, float* buf, int buf_floats,
                                         long long U, bool aborted) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NWARPS = NTHREADS / 32;
  const long long G = gridDim.x;
  const long long S = G + a.B;           // partial slots: CTA + sequence
  if (m->total_items == 0) return;     // nothing split or empty: no barrier, all CTAs agree
  // ---- grid barrier: all partials written before any is read
  if (tid == 0) {
    __threadfence();
    const unsigned int before = atomicAdd(a.sync, 1u);
    // the last CTA to arrive does not wait
    const bool ok = before + 1u >= static_cast<unsigned int>(G) ||
                    spin_until_geq(a.sync, static_cast<unsigned int>(G));
    __threadfence();
    if (!ok) {
      set_err(a.err, LSA_DEVERR_TIMEOUT);
      m->abort = 1;
    }
  }
  __syncthreads();
  fence_proxy_async_global();           // the partials are read back by bulk copies
  bool failed = m->abort != 0 || aborted;   // the same value in every thread
  const bool precut = m->precut != 0;
  uint32_t group_no = 0;                 // phases of merge_bar completed so far
  for (int round = 0; !failed; ++round) {
    if (round > 0) {
      __syncthreads();
      if (warp == 0) plan_merge(a, U, round * MAXITEMS, m, lane);
      __syncthreads();
    }
    const int nrec = m->n_items;
    if (nrec == 0) break;
    bool first = round == 0 && precut;   // the first group was cut before the barrier
    if (!first && tid == 0) {
      m->cur_rec = 0;
      m->cur_j = -1;
    }
    while (!failed) {
      if (tid == 0) {
        if (!first) cut_group(a, m, buf_floats);
        if (m->group_bytes > 0)
          mbar_arrive_expect_tx(&m->merge_bar, static_cast<uint32_t>(m->group_bytes));
      }
      first = false;
      __syncthreads();
      const int nr = m->n_runs;
      if (nr == 0) break;
      const bool copies = m->group_bytes > 0;
      // ---- one bulk copy per (run, chunk), spread over the threads
      {
        int q = 0, before = 0;
        for (int p = tid;; p += NTHREADS) {
          while (q < nr && p >= before + m->run_nch[q]) before += m->run_nch[q++];
          if (q >= nr) break;
          const int n = m->run_n[q];
          if (n == 0) continue;
          const int i = p - before;
          const long long b = m->run_b[q], h = m->run_h[q];
          const float* src = a.part_o + ((static_cast<long long>(m->run_c0[q] + i) * a.H + h) * S +
                                         m->run_clo[q] + b) * CW;
          bulk_load(buf + m->run_off[q] + static_cast<long long>(i) * n * CW, src,
                    static_cast<uint32_t>(n) * (CW * 4u), &m->merge_bar);
        }
      }
      // ---- and one bulk copy of each run's (m, l) quadruples
      for (int q = tid; q < nr; q += NTHREADS) {
        const int n = m->run_n[q];
        if (n == 0) continue;
        const float* src = a.part_ml + (static_cast<long long>(m->run_h[q]) * S + m->run_clo[q] +
                                        m->run_b[q]) * 4;
        bulk_load(buf + m->run_off[q] + static_cast<long long>(m->run_nch[q]) * n * CW, src,
                  static_cast<uint32_t>(n) * 16u, &m->merge_bar);
      }
      bool ok = true;
      if (copies) ok = mbar_wait(&m->merge_bar, group_no & 1, nullptr);
      if (copies) ++group_no;
      if (!__syncthreads_and(ok)) {
        if (tid == 0) {
          set_err(a.err, LSA_DEVERR_TIMEOUT);
          m->abort = 1;
        }
        failed = true;
        break;
      }
      // ---- split weights, one warp per run, from shared memory; an empty CTA's slot (no
      // units, nothing written; only possible when the grid has more CTAs than units)
      // gets weight 0. Each lane loads its up to MAX_GRID / 32 slots at once.
      for (int q = warp; q < nr; q += NWARPS) {
        const int n = m->run_n[q];
        const float* ml = buf + m->run_off[q] + static_cast<long long>(m->run_nch[q]) * n * CW;
        float* w = const_cast<float*>(ml) + 4 * n;
        const long long c0 = m->run_clo[q];
        constexpr int PER_LANE = MAX_GRID / 32;
        float mk[PER_LANE], lk[PER_LANE];
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
          const int k = lane + 32 * i;
          mk[i] = -INFINITY;
          lk[i] = 0.f;
          if (k < n && (U >= G || m->ustart[c0 + k] != m->ustart[c0 + k + 1])) {
            const float2 v = *reinterpret_cast<const float2*>(ml + 4 * k);
            mk[i] = v.x;
            lk[i] = v.y;
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) mx = fmaxf(mx, mk[i]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float ls = 0.f;
#pragma unroll
        for (int i = 0; i < PER_LANE; ++i) {
          const int k = lane + 32 * i;
          const float wk = mk[i] == -INFINITY ? 0.f : exp2f(mk[i] - mx);
          ls += wk == 0.f ? 0.f : wk * lk[i];
          if (k < n) w[k] = wk;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
        if (lane == 0) m->run_inv[q] = ls > 0.f ? 1.f / ls : 0.f;
      }
      __syncthreads();
      // ---- outputs: jobs are (run, chunk, 16-byte column); the threads of a slice take
      // consecutive columns and walk the same rows, slices split the rows in ranges
      int total_c4 = 0;
      for (int q = 0; q < nr; ++q) total_c4 += (CW / 4) * m->run_nch[q];
      int slices = NTHREADS / (total_c4 > 0 ? total_c4 : 1);
      slices = slices < 1 ? 1 : (slices > 8 ? 8 : slices);
      const int per_c = NTHREADS / slices;     // columns per pass
      const int sl = tid / per_c, t = tid - sl * per_c;
      float4* scratch = reinterpret_cast<float4*>(buf + m->group_floats);
      for (int base = 0; base < total_c4; base += per_c) {
        const int c4 = base + t;
        const bool act = sl < slices && c4 < total_c4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        int q = 0, i = 0, col = 0;
        if (act) {
          int x = c4;
          while (x >= (CW / 4) * m->run_nch[q]) x -= (CW / 4) * m->run_nch[q++];
          i = x / (CW / 4);
          col = x - i * (CW / 4);
          const int n = m->run_n[q];
          const int k0 = (sl * n) / slices, k1 = ((sl + 1) * n) / slices;
          const float* rows = buf + m->run_off[q] + static_cast<long long>(i) * n * CW + 4 * col;
          const float* w = buf + m->run_off[q] + static_cast<long long>(m->run_nch[q]) * n * CW + 4 * n;
          // a zero weight marks an empty CTA's row, never written: its bits are dropped.
          // Rows go four at a time (loads first, two accumulators), joined in fixed order.
          float4 acc2 = make_float4(0.f, 0.f, 0.f, 0.f);
          int k = k0;
          for (; k + 4 <= k1; k += 4) {
            float wv[4];
            float4 rv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              wv[e] = w[k + e];
              rv[e] = *reinterpret_cast<const float4*>(rows + static_cast<long long>(k + e) * CW);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float4& A = (e & 1) ? acc2 : acc;
              const bool z = wv[e] == 0.f;
              A.x = fmaf(wv[e], z ? 0.f : rv[e].x, A.x);
              A.y = fmaf(wv[e], z ? 0.f : rv[e].y, A.y);
              A.z = fmaf(wv[e], z ? 0.f : rv[e].z, A.z);
              A.w = fmaf(wv[e], z ? 0.f : rv[e].w, A.w);
            }
          }
          for (; k < k1; ++k) {
            const float wk = w[k];
            const float4 r = *reinterpret_cast<const float4*>(rows + static_cast<long long>(k) * CW);
            const bool z = wk == 0.f;
            acc.x = fmaf(wk, z ? 0.f : r.x, acc.x);
            acc.y = fmaf(wk, z ? 0.f : r.y, acc.y);
            acc.z = fmaf(wk, z ? 0.f : r.z, acc.z);
            acc.w = fmaf(wk, z ? 0.f : r.w, acc.w);
          }
          acc.x += acc2.x;
          acc.y += acc2.y;
          acc.z += acc2.z;
          acc.w += acc2.w;
        }
        if (sl < slices) scratch[tid] = acc;
        __syncthreads();
        if (act && sl == 0) {
          float4 tot = acc;
          for (int j = 1; j < slices; ++j) {
            const float4 v = scratch[j * per_c + t];
            tot.x += v.x;
            tot.y += v.y;
            tot.z += v.z;
            tot.w += v.w;
          }
          const float inv = m->run_inv[q];
          const __nv_bfloat162 p0 = __floats2bfloat162_rn(tot.x * inv, tot.y * inv);
          const __nv_bfloat162 p1 = __floats2bfloat162_rn(tot.z * inv, tot.w * inv);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t*>(&p0);
          pk.y = *reinterpret_cast<const uint32_t*>(&p1);
          *reinterpret_cast<uint2*>(a.out + (static_cast<long long>(m->run_b[q]) * a.H + m->run_h[q]) *
                                                a.d + (m->run_c0[q] + i) * CW + 4 * col) = pk;
        }
        __syncthreads();
      }
      __syncthreads();                  // the buffer is refilled by the next group
    }
    if (nrec < MAXITEMS) break;
  }
  // ---- departure: the last CTA out resets the counters for the next launch
  __syncthreads();
  if (tid == 0) {
    if (atomicAdd(a.sync + 1, 1u) == static_cast<unsigned int>(G) - 1u) {
      atomicExch(a.sync, 0u);
      atomicExch(a.sync + 1, 0u);
    }
  }
}

template <int HP, int NDC>
struct Layout {
  static constexpr int NDB = NDC / 2;                   // 128-dim blocks of O^T
  static constexpr int Q_BYTES = NDC * HP * 128;        // [NDC][HP][64] bf16
  static constexpr int RING_BYTES = NST * STAGE_BYTES;
  static constexpr int P_BYTES = 2 * HP * 128;          // [2][HP][64] bf16 (P^T, K-major)
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = Q_OFF + Q_BYTES;
  static constexpr int P_OFF = RING_OFF + RING_BYTES;
  static constexpr int MISC_OFF = P_OFF + P_BYTES;
  static constexpr int SMEM = MISC_OFF + static_cast<int>(sizeof(Misc)) + 1024;  // + alignment
  static constexpr int TMEM_USED = 2 * HP + NDB * HP;
  static constexpr uint32_t TMEM_COLS =
      TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(TMEM_USED <= 512, "tensor memory overflow");
  static_assert(NDC % 2 == 0 && NST % 2 == 0, "V stage pairs must not straddle the ring end");
  static_assert(HP % 16 == 0 && HP <= 64, "heads padded to 16, at most 64");
};

template <int HP, int NDC>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_splitk_kernel(const __grid_constant__ CUtensorMap map_kv,
                       const __grid_constant__ CUtensorMap map_q,
                       const __grid_constant__ Args a) {
  using LY = Layout<HP, NDC>;
  constexpr int NDB = LY::NDB;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived by pointer arithmetic on the shared array so the
  // compiler keeps addressing it as shared memory (no generic loads and stores)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + LY::Q_OFF;
  uint8_t* sRing = smem + LY::RING_OFF;
  uint8_t* sP = smem + LY::P_OFF;
  Misc* m = reinterpret_cast<Misc*>(smem + LY::MISC_OFF);
  volatile int* abort = &m->abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&m->full[i], 1);
      mbar_init(&m->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&m->s_full[i], 1);
      mbar_init(&m->s_free[i], 4);  // one arrive per softmax warp
    }
    mbar_init(&m->p_full, 4);
    mbar_init(&m->pv_done, 1);
    mbar_init(&m->q_full, 1);
    mbar_init(&m->q_free, 1);
    mbar_init(&m->mma_done, 1);
    mbar_init(&m->merge_bar, 1);
    m->abort = 0;
    m->precut = 0;
    m->resc_tile = -1;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_kv);
    prefetch_tensormap(&map_q);
  }
  if (warp == 1) {
    tmem_alloc(&m->tmem_base, LY::TMEM_COLS);
    tmem_relinquish();
  }
  // Launched as a programmatic dependent: everything above overlaps the previous
  // kernel's tail; nothing a preceding kernel may write is read before this point.
  grid_dependency_wait();
  grid_dependents_launch();
  long long U = 0;
  if (warp == 0) U = warp_total_units(a, lane);
  // grid-wide split of the batch's units
  const long long G = gridDim.x;
  long long us = 0, ue = 0;
  if (warp == 0) {
    us = (static_cast<long long>(blockIdx.x) * U) / G;
    ue = (static_cast<long long>(blockIdx.x + 1) * U) / G;
    plan_segments(a, us, ue, 0, m, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = m->tmem_base;

  // per-role pipeline counters (persist across segments and batches)
  int ring_pos = 0;      // stages armed (producer) / consumed (MMA) so far
  int seg_count = 0;     // segments started by this role
  int gtile_s = 0;       // S tiles issued / consumed
  int gtile_o = 0;       // PV tiles issued / P tiles produced
  const uint64_t evict_first = (warp == 0) ? l2_policy_evict_first() : 0ull;
  for (int batch = 0;; ++batch) {
    const int nseg = m->nseg;
    if (warp == 0 && a.k_new != nullptr) {
      // Fused append: the CTA that owns a sequence's last unit writes the step's token
      // into its tail page before this warp's TMA loads read that page.
      for (int g = 0; g < nseg; ++g) {
        const Seg sg = m->seg[g];
        if (sg.u1 != seq_units(a, sg.b)) continue;
        const int n = __ldg(a.n_entries + sg.b);
        const int page = __ldg(a.block_table + static_cast<long long>(sg.b) * a.bt_stride + n - 1);
        if (page < 0 || page >= a.n_pages) continue;  // reported by the producer
        const long long row = static_cast<long long>(page) * 128 + (a.fused_tail - 1);
        const uint4* ks = reinterpret_cast<const uint4*>(a.k_new + static_cast<long long>(sg.b) * a.d);
        const uint4* vs = reinterpret_cast<const uint4*>(a.v_new + static_cast<long long>(sg.b) * a.d);
        uint4* kd = reinterpret_cast<uint4*>(a.pool + row * a.d);
        uint4* vd = reinterpret_cast<uint4*>(a.pool + (row + 64) * a.d);
        for (int i = lane; i < a.d / 8; i += 32) {
          kd[i] = __ldg(ks + i);
          vd[i] = __ldg(vs + i);
        }
        if (lane == 0 && a.tail_len_out != nullptr) a.tail_len_out[sg.b] = a.fused_tail;
      }
      fence_proxy_async_global();
      __syncwarp();
    }
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        for (int g = 0; g < nseg && !*abort; ++g) {
          const Seg sg = m->seg[g];
          const int T = (sg.u1 - sg.u0 + 3) >> 2;
          if (seg_count > 0 && !mbar_wait(&m->q_free, (seg_count - 1) & 1, abort)) break;
          mbar_arrive_expect_tx(&m->q_full, NDC * a.H * 128);
          for (int c = 0; c < NDC; ++c)
            tma_load_2d(sQ + c * HP * 128, &map_q, &m->q_full, 64 * c, sg.b * a.H);
          ++seg_count;
          const int32_t* bt = a.block_table + static_cast<long long>(sg.b) * a.bt_stride;
          for (int i = 0; i <= T && !*abort; ++i) {
            for (int kv = 0; kv < 2; ++kv) {
              // stage order per step i: K of tile i, then V of tile i-1
              const int tile = kv == 0 ? i : i - 1;
              if (tile < 0 || tile >= T) continue;
              int tu0, tu1;
              tile_range(sg, tile, tu0, tu1);
              int ys[4];
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int u = tu0 + r;
                // rows past the tile's units: a box outside the map, zero-filled by the
                // copy engine without reading memory (the softmax masks those rows)
                const int page = u < tu1 ? __ldg(bt + (u >> 1)) : -1;
                int y;
                if (u >= tu1) {
                  y = static_cast<int>(a.n_pages * 128);
                } else if (page < 0 || page >= a.n_pages) {
                  set_err(a.err, LSA_DEVERR_BAD_PAGE);
                  y = static_cast<int>(a.n_pages * 128);  // outside the map: zero fill
                } else {
                  y = page * 128 + kv * 64 + (u & 1) * UNIT;
                }
                ys[r] = y;
              }
              for (int c = 0; c < NDC; ++c) {
                const int st = ring_pos % NST;
                if (!mbar_wait(&m->empty[st], ((ring_pos / NST) & 1) ^ 1, abort)) break;
                mbar_arrive_expect_tx(&m->full[st], STAGE_BYTES);
                uint8_t* dst = sRing + st * STAGE_BYTES;
#pragma unroll
                for (int r = 0; r < 4; ++r)
                  tma_load_2d_hint(dst + r * (UNIT * 128), &map_kv, &m->full[st], 64 * c, ys[r],
                                   evict_first);
                ++ring_pos;
              }
            }
          }
        }
      }
      __syncwarp();
      if (!m->more) {
        // the producer's last loads are out: plan the fused merge and cut its first
        // group of runs meanwhile
        for (int c = lane; c <= G; c += 32) m->ustart[c] = (c * U) / G;
        plan_merge(a, U, 0, m, lane);
        __syncwarp();
        if (lane == 0 && m->total_items > 0 && m->n_items > 0) {
          m->cur_rec = 0;
          m->cur_j = -1;
          cut_group(a, m, LY::MISC_OFF / 4);
          m->precut = 1;
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t IDESC_S = idesc_bf16_f32(128, HP, false, false);
        constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HP, true, false);
        const uint32_t q_base = smem_u32(sQ), p_base = smem_u32(sP), ring_base = smem_u32(sRing);
        for (int g = 0; g < nseg && !*abort; ++g) {
          const Seg sg = m->seg[g];
          const int T = (sg.u1 - sg.u0 + 3) >> 2;
          if (!mbar_wait(&m->q_full, seg_count & 1, abort)) break;
          tc_fence_after();
          ++seg_count;
          bool ok = true;
          for (int i = 0; i <= T && ok; ++i) {
            if (i < T) {
              const int sb = gtile_s & 1;
              if (gtile_s >= 2 && !mbar_wait(&m->s_free[sb], ((gtile_s >> 1) - 1) & 1, abort)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t d_s = tmem + sb * HP;
              for (int kb = 0; kb < NDC && ok; ++kb) {
                const int stg = ring_pos % NST;
                if (!mbar_wait(&m->full[stg], (ring_pos / NST) & 1, abort)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint32_t st = ring_base + stg * STAGE_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  umma_bf16(d_s, sdesc_sw128(st + kk * 32, 16, 1024),
                            sdesc_sw128(q_base + kb * HP * 128 + kk * 32, 16, 1024), IDESC_S,
                            (kb | kk) != 0);
                umma_commit(&m->empty[stg]);
                ++ring_pos;
              }
              if (!ok) break;
              umma_commit(&m->s_full[sb]);
              if (i == T - 1) umma_commit(&m->q_free);
              ++gtile_s;
            }
            if (i >= 1) {
              const int j = i - 1;
              if (!mbar_wait(&m->p_full, gtile_o & 1, abort)) {
                ok = false;
                break;
              }
              tc_fence_after();
              for (int db = 0; db < NDB && ok; ++db) {
                const int st0 = ring_pos % NST;  // even: the pair (st0, st0+1) is adjacent
                if (!mbar_wait(&m->full[st0], (ring_pos / NST) & 1, abort) ||
                    !mbar_wait(&m->full[st0 + 1], (ring_pos / NST) & 1, abort)) {
                  ok = false;
                  break;
                }
                tc_fence_after();
                const uint32_t st = ring_base + st0 * STAGE_BYTES;
                const uint32_t d_o = tmem + 2 * HP + db * HP;
#pragma unroll
                for (int kk = 0; kk < TILE / 16; ++kk)
                  umma_bf16(d_o, sdesc_sw128(st + kk * 16 * 128, STAGE_BYTES, 1024),
                            sdesc_sw128(p_base + (kk >> 2) * HP * 128 + (kk & 3) * 32, 16, 1024),
                            IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&m->empty[st0]);
                umma_commit(&m->empty[st0 + 1]);
                ring_pos += 2;
              }
              if (!ok) break;
              umma_commit(&m->pv_done);
              ++gtile_o;
            }
          }
        }
      }
    } else {
      // ---------------------------------------------------------------- softmax
      // Every wait result is folded into the next barrier-with-reduction, so the four
      // warps always leave together and no named barrier is left half-arrived.
      const int sw = warp & 3;                 // TMEM sub-partition: rows [32*sw, 32*sw+32)
      const int t128 = tid - 64;               // 0..127
      const int row = sw * 32 + lane;          // token row of the tile
      const uint32_t lane_addr = static_cast<uint32_t>(sw * 32) << 16;
      bool failed = false;
      for (int g = 0; g < nseg && !failed; ++g) {
        const Seg sg = m->seg[g];
        const int T = (sg.u1 - sg.u0 + 3) >> 2;
        const int n_ent = __ldg(a.n_entries + sg.b);
        const int tl = seq_tail(a, sg.b);
        float m_run = -INFINITY;               // running max (log2 units) of head t128
        float lp[HP];
#pragma unroll
        for (int h = 0; h < HP; ++h) lp[h] = 0.f;
        for (int j = 0; j < T; ++j) {
          const int sb = gtile_s & 1;
          if (!failed) failed = !__all_sync(0xffffffffu, mbar_wait(&m->s_full[sb], (gtile_s >> 1) & 1, abort));
          tc_fence_after();
          // validity of this row's token
          int tu0, tu1;
          tile_range(sg, j, tu0, tu1);
          const int u = tu0 + sw;
          bool valid = u < tu1;
          if (valid && (u >> 1) == n_ent - 1) valid = (u & 1) * UNIT + lane < tl;
          // per-head tile max
          if (!failed) {
            float x[HP];
            tmem_ld_row<HP>(tmem + lane_addr + sb * HP, x);
            tmem_wait_ld();
            if (!__all_sync(0xffffffffu, valid)) {
#pragma unroll
              for (int h = 0; h < HP; ++h) x[h] = valid ? x[h] : -INFINITY;
            }
            warp_reduce_scatter<HP, true>(x, lane);
            store_scattered<HP>(m->red[sw], x, lane);
          }
          if (named_bar_any(1, 128, failed)) {
            failed = true;
            break;
          }
          if (t128 < HP) {
            const int h = t128;
            float mt = fmaxf(fmaxf(m->red[0][h], m->red[1][h]), fmaxf(m->red[2][h], m->red[3][h]));
            mt *= a.scale_log2;
            float al = 1.f;
            if (h < a.H && mt > m_run + RESCALE_LOG2) {
              al = exp2f(m_run - mt);          // 0 when nothing was accumulated yet
              m_run = mt;
              m->resc_tile = gtile_s;          // the same value from every head that rescales
            }
            m->m_use[h] = m_run;
            m->alpha[h] = al;
          }
          named_bar_sync(1, 128);
          float s[HP];
          tmem_ld_row<HP>(tmem + lane_addr + sb * HP, s);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&m->s_free[sb]);
          ++gtile_s;
          // gtile_s was advanced above: the tile whose alphas were just set is gtile_s - 1
          const bool rescale = m->resc_tile == gtile_s - 1;
          // The denominator sums the same bf16-rounded weights that multiply V, so the
          // output stays a normalised average of V rows (exact for a one-hot softmax); the
          // rounded bits are kept for the P operand.
          if (!rescale && a.H == HP && __all_sync(0xffffffffu, valid)) {
            // common case: no head rescales, every row and head is live
#pragma unroll
            for (int h = 0; h < HP; h += 2) {
              const float p0 = ex2_approx(fmaf(s[h], a.scale_log2, -m->m_use[h]));
              const float p1 = ex2_approx(fmaf(s[h + 1], a.scale_log2, -m->m_use[h + 1]));
              // both weights rounded by one conversion: p0 in the low half, p1 in the high
              const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
              const uint32_t w = *reinterpret_cast<const uint32_t*>(&pb);
              lp[h] += __uint_as_float(w << 16);
              lp[h + 1] += __uint_as_float(w & 0xffff0000u);
              s[h] = __uint_as_float(w & 0xffffu);
              s[h + 1] = __uint_as_float(w >> 16);
            }
          } else {
#pragma unroll
            for (int h = 0; h < HP; ++h) {
              const float mu = m->m_use[h];
              const float al = m->alpha[h];
              const float p = (valid && h < a.H) ? ex2_approx(fmaf(s[h], a.scale_log2, -mu)) : 0.f;
              const __nv_bfloat16 pb = __float2bfloat16_rn(p);
              lp[h] = lp[h] * al + __bfloat162float(pb);
              s[h] = __uint_as_float(static_cast<uint32_t>(__bfloat16_as_ushort(pb)));
            }
          }
          // the previous tile's P . V must be done before P is overwritten or O rescaled
          if (gtile_o >= 1)
            failed = !__all_sync(0xffffffffu, mbar_wait(&m->pv_done, (gtile_o - 1) & 1, abort));
          if (failed) continue;                // the next barrier reports it to all warps
          tc_fence_after();
          if (rescale && j > 0) {
#pragma unroll
            for (int db = 0; db < NDB; ++db) {
#pragma unroll
              for (int c = 0; c < HP / 16; ++c) {
                const uint32_t ta = tmem + lane_addr + 2 * HP + db * HP + 16 * c;
                float o[16];
                tmem_ld16(ta, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] *= m->alpha[16 * c + i];
                tmem_st16(ta, o);
              }
            }
            tmem_wait_st();
          }
          // P^T (K-major: row = head, 128 tokens in two 64-token chunks), bf16
          {
            uint8_t* pc = sP + (row >> 6) * HP * 128;
            const uint32_t byte_in_row = (row & 63) * 2;
#pragma unroll
            for (int h = 0; h < HP; ++h)
              *reinterpret_cast<uint16_t*>(pc + sw128_offset(h, byte_in_row)) =
                  static_cast<uint16_t>(__float_as_uint(s[h]));
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&m->p_full);
          ++gtile_o;
        }
        if (named_bar_any(1, 128, failed)) {
          failed = true;
          break;
        }
        // ------------------------------------------------------- segment epilogue
        failed = !__all_sync(0xffffffffu, mbar_wait(&m->pv_done, (gtile_o - 1) & 1, abort));
        tc_fence_after();
        if (!failed) {
          warp_reduce_scatter<HP, false>(lp, lane);
          store_scattered<HP>(m->red[sw], lp, lane);
        }
        if (named_bar_any(1, 128, failed)) {
          failed = true;
          break;
        }
        // a sequence held whole by this CTA is normalised and written out here; a split
        // one leaves its partial (O, m, l) in slot CTA + sequence for the merge
        const bool whole = sg.u0 == 0 && sg.u1 == seq_units(a, sg.b);
        // the CTA's last segment: Q and the ring are idle, so a whole sequence's output is
        // staged there and written with bulk copies instead of per-thread scalar stores
        const bool staged = g == nseg - 1 && !m->more;
        const long long S = static_cast<long long>(gridDim.x) + a.B;
        const long long slot = static_cast<long long>(blockIdx.x) + sg.b;
        if (t128 < a.H) {
          const int h = t128;
          const float l = m->red[0][h] + m->red[1][h] + m->red[2][h] + m->red[3][h];
          if (whole) {
            m->alpha[h] = 1.f / l;
          } else {
            *reinterpret_cast<float4*>(a.part_ml + (h * S + slot) * 4) = make_float4(m_run, l, 0.f, 0.f);
          }
        }
        if (whole) named_bar_sync(1, 128);
        uint16_t* fo = a.out + static_cast<long long>(sg.b) * a.H * a.d;
        // staged: each 128-dim block is laid out [head][128] in its own region of the idle
        // ring / Q buffers; right after a block is complete, one thread per head stores
        // that head's row with a 1-D bulk copy, overlapping the staging of the next block
        const int esz = whole ? 2 : 4;
        const uint32_t blk_bytes = static_cast<uint32_t>(a.H) * 128u * esz;
        bool issued = false;
#pragma unroll 1
        for (int db = 0; db < NDB; ++db) {
          float ob[HP];
          tmem_ld_row<HP>(tmem + lane_addr + 2 * HP + db * HP, ob);
          tmem_wait_ld();
          const int col = db * 128 + row;       // this thread's head-dimension index
          // the partial's rows: chunk db of head h in slot `slot` is 128 contiguous floats
          float* po = a.part_o + (static_cast<long long>(db) * a.H * S + slot) * CW;
          if (staged) {
            const uint32_t base = smem_u32(smem) + db * blk_bytes + row * esz;
            if (whole) {
#pragma unroll
              for (int h = 0; h < HP; ++h)
                if (h < a.H) {
                  const __nv_bfloat16 v = __float2bfloat16_rn(ob[h] * m->alpha[h]);
                  st_shared_u16(base + h * 256u, *reinterpret_cast<const uint16_t*>(&v));
                }
            } else {
#pragma unroll
              for (int h = 0; h < HP; ++h)
                if (h < a.H) st_shared_f32(base + h * 512u, ob[h]);
            }
            if (whole) fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (whole) {
              if (t128 < a.H) {
                const uint8_t* src = smem + db * blk_bytes + t128 * 256u;
                bulk_store(fo + static_cast<long long>(t128) * a.d + db * 128, src, 256u);
                issued = true;
              }
            } else {
              // each warp copies whole 512-byte head rows: one 16-byte piece per lane
              const float4* src = reinterpret_cast<const float4*>(smem + db * blk_bytes);
              for (int h = sw; h < a.H; h += 4)
                reinterpret_cast<float4*>(po + static_cast<long long>(h) * S * CW)[lane] = src[h * 32 + lane];
            }
          } else if (whole) {
#pragma unroll
            for (int h = 0; h < HP; ++h)
              if (h < a.H) {
                const __nv_bfloat16 v = __float2bfloat16_rn(ob[h] * m->alpha[h]);
                fo[static_cast<long long>(h) * a.d + col] = *reinterpret_cast<const uint16_t*>(&v);
              }
          } else {
            // for each head a warp writes 32 consecutive floats of the row (128 bytes)
#pragma unroll
            for (int h = 0; h < HP; ++h)
              if (h < a.H) po[static_cast<long long>(h) * S * CW + row] = ob[h];
          }
        }
        if (issued) {
          bulk_commit_and_wait();
          fence_proxy_async_global();
        }
        tc_fence_before();
        named_bar_sync(1, 128);
      }
    }

    // ------------------------------------------------------------ next batch
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!m->more || *abort) break;
    __syncthreads();
    if (warp == 0) plan_segments(a, us, ue, (batch + 1) * MAXSEG, m, lane);
    __syncthreads();
  }

  // ---------------------------------------------------------------- teardown
  if (*abort) {
    if (tid == 0) set_err(a.err, LSA_DEVERR_TIMEOUT);
    // the producer waits (bounded) for its own copies still in flight
    if (warp == 0 && lane == 0) {
      for (int k = max(0, ring_pos - NST); k < ring_pos; ++k)
        mbar_wait(&m->full[k % NST], (k / NST) & 1, nullptr);
      if (seg_count > 0) mbar_wait(&m->q_full, (seg_count - 1) & 1, nullptr);
    }
    // the MMA thread waits (bounded) for its own tensor-core work
    if (warp == 1 && lane == 0) {
      umma_commit(&m->mma_done);
      mbar_wait(&m->mma_done, 0, nullptr);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, LY::TMEM_COLS);
  // ring, Q and P buffers are free now: the merge reuses them
  {
    __shared__ long long s_U;
    if (tid == 0) s_U = U;
    __syncthreads();
    merge_phase(a, m, reinterpret_cast<float*>(smem), LY::MISC_OFF / 4, s_U, *abort != 0);
  }
}

}  // namespace attn
}  // namespace lsa

// ------------------------------------------------------------------------ host side
namespace {

using lsa::attn::Args;

// Workspace: the two grid-barrier counters on their own 256-byte line, then fp32
// partial O [d/128][H][G+B][128] and partial (m, l, pad, pad) [H][G+B][4].
size_t attn_ws_bytes(int B, int H, int d, int n_sm) {
  const size_t slots = static_cast<size_t>(n_sm) + static_cast<size_t>(B);
  const size_t body = slots * static_cast<size_t>(H) * (static_cast<size_t>(d) + 4) * sizeof(float);
  return (body + 255) / 256 * 256 + 256;
}

// Per-device launch state of one kernel instantiation: whether the device accepts a
// cooperative launch that is also a programmatic dependent. Kept per device (a process
// may drive several GPUs from several host threads).
struct LaunchState {
  std::atomic<int> pdl{1};        // 0: this device refused PDL with a cooperative launch
};
constexpr int MAX_DEVICES = 64;

template <int HP, int NDC>
lsa_status launch_attn(const CUtensorMap& mkv, const CUtensorMap& mq, const Args& a, int G,
                       cudaStream_t stream) {
  using LY = lsa::attn::Layout<HP, NDC>;
  auto kern = lsa::attn::attn_splitk_kernel<HP, NDC>;
  static LaunchState state[MAX_DEVICES];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return LSA_ERR_CUDA;
  LaunchState& ls = state[dev];
  const lsa_status st = lsa_host::ensure_smem_limit(reinterpret_cast<const void*>(kern), LY::SMEM);
  if (st != LSA_OK) return st;
  // Cooperative launch: all G CTAs (one per SM) are resident together, which the
  // fused merge's grid barrier relies on.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(lsa::attn::NTHREADS);
  cfg.dynamicSmemBytes = LY::SMEM;
  cfg.stream = stream;
  // Programmatic stream serialisation lets this launch's CTAs set up while the previous
  // kernel in the stream drains; the kernel waits for it before touching any data.
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  const bool pdl = ls.pdl.load(std::memory_order_relaxed) != 0;
  cfg.numAttrs = pdl ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mkv, mq, a);
  if (e == cudaSuccess) return LSA_OK;
  cudaGetLastError();
  // Only the answer "not supported" to the attribute combination turns PDL off (for this
  // device, for good); any other failure is reported to the caller as it is.
  if (!pdl || e != cudaErrorNotSupported) return LSA_ERR_CUDA;
  ls.pdl.store(0, std::memory_order_relaxed);
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, mkv, mq, a) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

template <int HP>
lsa_status dispatch_d(const CUtensorMap& mkv, const CUtensorMap& mq, const Args& a, int G,
                      cudaStream_t s) {
  switch (a.d) {
    case 128: return launch_attn<HP, 2>(mkv, mq, a, G, s);
    case 256: return launch_attn<HP, 4>(mkv, mq, a, G, s);
    case 384: return launch_attn<HP, 6>(mkv, mq, a, G, s);
    case 512: return launch_attn<HP, 8>(mkv, mq, a, G, s);
    default: return LSA_ERR_INVALID_ARG;
  }
}

}  // namespace

namespace lsa_host {

// Host checks of every argument of a decode-attention call except the workspace.
lsa_status check_attn_args(const uint16_t* q, const uint16_t* hbm_pool, int64_t n_pages,
                           const int32_t* block_table, int32_t bt_stride,
                           const int32_t* n_entries, const int32_t* tail_len, int32_t B,
                           int32_t H, int32_t d, float scale, const uint16_t* out,
                           const int32_t* err, const AppendArgs* append) {
  if (!q || !hbm_pool || !block_table || !n_entries || !out || !err) return LSA_ERR_INVALID_ARG;
  if (!append && !tail_len) return LSA_ERR_INVALID_ARG;
  if (append && (!append->k_new || !append->v_new || append->tail < 1 || append->tail > 64))
    return LSA_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || H > 64 || bt_stride <= 0 || n_pages <= 0) return LSA_ERR_INVALID_ARG;
  if (d != 128 && d != 256 && d != 384 && d != 512) return LSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return LSA_ERR_INVALID_ARG;
  if (n_pages > (int64_t(1) << 23)) return LSA_ERR_INVALID_ARG;  // page rows must fit in int32
  if (static_cast<int64_t>(B) * H > (int64_t(1) << 30)) return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(hbm_pool) |
       reinterpret_cast<uintptr_t>(out)) & 15u)
    return LSA_ERR_INVALID_ARG;
  if (append && ((reinterpret_cast<uintptr_t>(append->k_new) |
                  reinterpret_cast<uintptr_t>(append->v_new)) & 15u))
    return LSA_ERR_INVALID_ARG;
  return LSA_OK;
}

lsa_status decode_attn(const uint16_t* q, const uint16_t* hbm_pool, int64_t n_pages,
                       const int32_t* block_table, int32_t bt_stride, const int32_t* n_entries,
                       const int32_t* tail_len, int32_t B, int32_t H, int32_t d, float scale,
                       uint16_t* out, void* ws, size_t ws_bytes, int32_t* err, void* stream,
                       const AppendArgs* append) {
  lsa_host::NvtxRange nvtx_range("lsa_decode_attn");
  lsa_status st0 = check_attn_args(q, hbm_pool, n_pages, block_table, bt_stride, n_entries,
                                   tail_len, B, H, d, scale, out, err, append);
  if (st0 != LSA_OK) return st0;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u)) return LSA_ERR_INVALID_ARG;
  const int G = sm_count();
  if (G <= 0) return LSA_ERR_CUDA;
  if (G > lsa::attn::MAX_GRID) return LSA_ERR_UNIMPLEMENTED;
  if (ws_bytes < attn_ws_bytes(B, H, d, G)) return LSA_ERR_INVALID_ARG;
  const int HP = (H + 15) / 16 * 16;
  const int HPk = HP <= 16 ? 16 : HP <= 32 ? 32 : 64;

  CUtensorMap mkv, mq;
  lsa_status st = encode_tiled_2d(&mkv, hbm_pool, d, static_cast<uint64_t>(n_pages) * 128,
                                  static_cast<uint64_t>(d) * 2, 64, lsa::attn::UNIT,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != LSA_OK) return st;
  st = encode_tiled_2d(&mq, q, d, static_cast<uint64_t>(B) * H, static_cast<uint64_t>(d) * 2, 64,
                       H, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != LSA_OK) return st;

  Args a = {};
  a.block_table = block_table;
  a.n_entries = n_entries;
  a.tail_len = tail_len;
  // the barrier counters sit at a fixed place (the first 256 bytes) whatever the shape,
  // so one array can serve calls of different shapes in turn
  a.sync = static_cast<unsigned int*>(ws);
  a.part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + 256);
  a.part_ml = a.part_o + (static_cast<size_t>(G) + B) * H * d;
  a.out = out;
  a.pool = const_cast<uint16_t*>(hbm_pool);
  if (append) {
    a.k_new = append->k_new;
    a.v_new = append->v_new;
    a.tail_len_out = append->tail_len_out;
    a.fused_tail = append->tail;
  }
  a.err = err;
  a.n_pages = n_pages;
  a.bt_stride = bt_stride;
  a.B = B;
  a.H = H;
  a.d = d;
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (HPk) {
    case 16: return dispatch_d<16>(mkv, mq, a, G, s);
    case 32: return dispatch_d<32>(mkv, mq, a, G, s);
    default: return dispatch_d<64>(mkv, mq, a, G, s);
  }
}

}  // namespace lsa_host

extern "C" size_t lsa_decode_attn_workspace_size(int32_t B, int32_t H, int32_t d, int32_t n_sm) {
  if (B <= 0 || H <= 0 || d <= 0 || n_sm <= 0) return 0;
  return attn_ws_bytes(B, H, d, n_sm);
}

extern "C" lsa_status lsa_decode_attn(const uint16_t* q, const uint16_t* hbm_pool, int64_t n_pages,
                                      const int32_t* block_table, int32_t bt_stride,
                                      const int32_t* n_entries, const int32_t* tail_len,
                                      int32_t B, int32_t H, int32_t d, float scale, uint16_t* out,
                                      void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  return lsa_host::decode_attn(q, hbm_pool, n_pages, block_table, bt_stride, n_entries, tail_len,
                               B, H, d, scale, out, ws, ws_bytes, err, stream, nullptr);
}

// ------------------------------------------------- decode attention without allocation
// For callers that cannot allocate device memory at all, e.g. code running inside a
// host framework that owns every allocation, a real-time loop that must not call into
// the CUDA allocator, or a plugin that receives only input and output buffers: the split
// partials and the merge barrier counters live in one fixed device array of this library.
// Every call shares the array, so calls that overlap on the GPU race with one another.
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LSA_NOALLOC_SCRATCH_BYTES];

struct NoallocScratch {
  void* ptr = nullptr;
  bool ready = false;
};

std::mutex g_noalloc_mutex;
NoallocScratch g_noalloc[64];

// Device address of the scratch array on the current device. In host code the array's
// name is only a host-side stand-in, so the address is looked up once per device, with
// that device current. That first time, a clear of the array's first 256 bytes (the
// merge barrier counters; partials are always written before they are read) is enqueued
// on the caller's stream, so it is ordered before the kernel launched next on the same
// stream. (Global device variables without an initialiser also start at zero.)
lsa_status noalloc_scratch(void** out, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoallocScratch& s = g_noalloc[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return LSA_ERR_CUDA;
    }
    if (cudaMemsetAsync(p, 0, 256, stream) != cudaSuccess) {
      cudaGetLastError();
      return LSA_ERR_CUDA;
    }
    s.ptr = p;
    s.ready = true;
  }
  *out = s.ptr;
  return LSA_OK;
}

}  // namespace

extern "C" lsa_status lsa_decode_attn_noalloc(const uint16_t* q, const uint16_t* hbm_pool,
                                              int64_t n_pages, const int32_t* block_table,
                                              int32_t bt_stride, const int32_t* n_entries,
                                              const int32_t* tail_len, int32_t B, int32_t H,
                                              int32_t d, float scale, uint16_t* out,
                                              int32_t* err, void* stream) {
  // the arguments first, so that a malformed call is told so and not that it is too big
  const lsa_status chk = lsa_host::check_attn_args(q, hbm_pool, n_pages, block_table, bt_stride,
                                                   n_entries, tail_len, B, H, d, scale, out, err,
                                                   nullptr);
  if (chk != LSA_OK) return chk;
  const int G = lsa_host::sm_count();
  if (G <= 0) return LSA_ERR_CUDA;
  const size_t need = attn_ws_bytes(B, H, d, G);
  if (need > static_cast<size_t>(LSA_NOALLOC_SCRATCH_BYTES)) return LSA_ERR_CAPACITY;
  void* ws = nullptr;
  const lsa_status st = noalloc_scratch(&ws, static_cast<cudaStream_t>(stream));
  if (st != LSA_OK) return st;
  return lsa_host::decode_attn(q, hbm_pool, n_pages, block_table, bt_stride, n_entries, tail_len,
                               B, H, d, scale, out, ws, need, err, stream, nullptr);
}
