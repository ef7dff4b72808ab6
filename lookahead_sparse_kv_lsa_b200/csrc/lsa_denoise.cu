// Label denoising of the indexer's training targets ("FlashMemory-DeepSeek-V4 Explained",
// zhichai.net, section 3 "Label Denoising Pipeline"): for every token window and every
// CSA layer, a softmax over the layer's raw Lightning-Indexer logits of all KV blocks;
// the smallest set of blocks whose probabilities reach top_p (0.6 on the page); then a
// block is a label of the window when at least min_votes (3 of the 21) layers kept it.
//
// One CTA per (window, layer) row, the row in shared memory. The top-p set is found
// without sorting the row:
//   1. row max M, then e_i = 2^(x_i*log2(e) - M*log2(e)) for every block; a 16-bin
//      histogram of the mass by whole logit units below M gives the total S and the bin
//      j0 where the running mass from the top crosses T = top_p * S;
//   2. one pass writes the mask words of the blocks above bin j0 (kept whatever the
//      boundary) and appends the blocks of bin j0 to a candidate list, one segment per
//      warp, without atomics;
//   3. the list is split 16 ways, linearly in the order-preserving integer key of the
//      logit, until at most 256 candidates remain; they are ranked by (logit descending,
//      id ascending), their mass is scanned in that order in fp64, and the first rank
//      whose running mass reaches T fixes the last kept (logit, id) pair. When all the
//      remaining candidates share one logit, the first m of them by id are kept, m the
//      smallest count whose mass reaches T;
//   4. the kept list entries are OR-ed into the mask words.
// When bin j0 holds more blocks than the list, the bin itself is split over the row
// first and the mask is then derived from the row. Ordering uses the exact fp32
// logits, so blocks with equal probability are the blocks with equal logits and they
// are taken by increasing id; only the position of the boundary depends on rounding
// (fp32 e_i, fp64 sums).
//
// Each thread accumulates its share of a histogram in its own shared-memory column
// (bank = lane), so no shared atomics are needed for the mass; the bins are then summed
// in fp64. The vote runs in the last CTA of each window (a per-window ticket in the
// workspace), as bit-sliced counters over the layers' 32-block mask words.
#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int NT = 256;               // threads per CTA
constexpr int NWARP = NT / 32;
constexpr int DN_BINS = 16;
constexpr int DN_CAND = 256;          // candidates resolved by ranking
constexpr int DN_MAX_REFINE = 12;     // key-range splits; 9 always suffice for 32-bit keys
constexpr int DN_PLANES = 6;          // vote counter bit planes: counts up to 63 layers
constexpr int DN_LIST = 2048;         // candidate list
constexpr int DN_SEG = DN_LIST / NWARP;  // one list segment per warp
constexpr int DN_SLOTS = DN_LIST / NT;   // list slots per thread
constexpr float DN_LOG2E = 1.4426950408889634f;

struct DenoiseArgs {
  const float* logits;   // [W][L][N]
  int32_t W, L, N, NW;   // NW = ceil(N / 32)
  double top_p;
  int32_t min_votes;
  uint32_t* set_mask;    // [W][L][NW]
  int32_t* set_cnt;      // [W][L] or null
  uint32_t* label_mask;  // [W][NW] or null
  int32_t* label_ids;    // [W][label_cap]
  int32_t label_cap;
  int32_t* label_cnt;    // [W]
  uint32_t* tickets;     // [W], zero between calls
  int32_t* err;
};

// Shared memory: this fixed part, then the row (NW * 32 floats), then NW mask words.
struct Smem {
  float hist[DN_BINS * NT];  // per-thread columns; later tie words
  uint32_t lk[DN_LIST];      // candidate list keys, segment w at [w * DN_SEG, ...)
  int32_t li[DN_LIST];       // and block ids
  double bsum[DN_BINS];
  double wsum[NWARP];
  double se[DN_CAND];        // candidate mass in rank order
  uint32_t ckey[DN_CAND];    // candidates, in arrival order
  int32_t cid[DN_CAND];
  int32_t spos[DN_CAND];     // rank -> arrival slot
  int32_t cw[NWARP];         // entries per list segment (more than DN_SEG: overflow)
  float wmax[NWARP];
  int32_t wcnt[NWARP];
  int32_t c;                 // elements matched by the last compaction
  uint32_t kmin, kmax;       // key range of those elements
  int32_t pick;              // rank of the last kept candidate
  uint32_t tau_key;          // the last kept (key, id)
  int32_t tau_id;
  int32_t last;              // this CTA closes its window
  int32_t total;
  int32_t pad[3];
};
static_assert(sizeof(Smem) % 16 == 0, "the row starts 16-byte aligned");

extern __shared__ __align__(16) unsigned char dn_smem[];
__device__ __forceinline__ Smem& sm() { return *reinterpret_cast<Smem*>(dn_smem); }
__device__ __forceinline__ float* row_x() { return reinterpret_cast<float*>(dn_smem + sizeof(Smem)); }
__device__ __forceinline__ uint32_t* row_words(int NW) {
  return reinterpret_cast<uint32_t*>(row_x() + static_cast<size_t>(NW) * 32);
}

// Order-preserving map of an fp32 value to uint32 (-0 taken as +0).
__device__ __forceinline__ uint32_t order_key(float v) {
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// 2^y on the special-function unit (relative error about 2^-22; results below 2^-126
// flush to zero, which removes mass under 1e-38 of the row maximum's).
__device__ __forceinline__ float pow2(float y) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
  return r;
}

// Probability mass of one block up to the row's common factor 1/S.
__device__ __forceinline__ float mass(float v, float ml2) { return pow2(fmaf(v, DN_LOG2E, -ml2)); }

// Which elements a pass looks at: the first pass's unit bin jsel below the max, or a
// key range [ka, kb] split into 16 linear key bins of which bin jsel is taken.
struct Pred {
  bool first;    // true: bin0(v) == jsel
  float M;
  uint32_t ka, kb;
  uint64_t mul;  // floor(16 * 2^32 / (kb - ka + 1))
  int jsel;      // -1: the whole key range
};

__device__ __forceinline__ int bin0(float v, float M) {
  return max(0, min(static_cast<int>(M - v), DN_BINS - 1));  // M - v >= 0 when finite
}
__device__ __forceinline__ int bin_key(uint32_t key, uint32_t kb, uint64_t mul) {
  return static_cast<int>((static_cast<uint64_t>(kb - key) * mul) >> 32);
}
__device__ __forceinline__ bool pred_in(const Pred& p, float v, uint32_t key) {
  if (p.first) return bin0(v, p.M) == p.jsel;
  if (key < p.ka || key > p.kb) return false;
  return p.jsel < 0 || bin_key(key, p.kb, p.mul) == p.jsel;
}
__device__ __forceinline__ Pred key_split(float M, uint32_t ka, uint32_t kb) {
  const uint64_t R = static_cast<uint64_t>(kb - ka) + 1ull;
  return Pred{false, M, ka, kb, (static_cast<uint64_t>(DN_BINS) << 32) / R, -1};
}

// Sum the NT per-thread histogram columns into s.bsum[] in fp64 (NT / 16 threads per bin).
__device__ void reduce_bins() {
  Smem& s = sm();
  constexpr int TPB = NT / DN_BINS;
  const int tid = threadIdx.x;
  const int b = tid / TPB, part = tid % TPB;
  double v = 0.0;
#pragma unroll 4
  for (int k = 0; k < NT / TPB; ++k) v += s.hist[b * NT + part + TPB * k];
#pragma unroll
  for (int o = TPB / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (part == 0) s.bsum[b] = v;
  __syncthreads();
}

// Scanning the bins from the top, the first non-empty bin where acc + the running mass
// reaches T (the last non-empty bin when rounding leaves the total short of T). acc
// becomes the mass above the chosen bin. Every thread computes the same answer.
__device__ int choose_bin(double T, double& acc) {
  const double* bsum = sm().bsum;
  double cum = acc, acc_last = acc;
  int last_nz = -1;
  for (int j = 0; j < DN_BINS; ++j) {
    const double bj = bsum[j];
    if (bj > 0.0) {
      if (cum + bj >= T) { acc = cum; return j; }
      last_nz = j;
      acc_last = cum;
    }
    cum += bj;
  }
  acc = acc_last;
  return last_nz < 0 ? 0 : last_nz;
}

// Warp-aggregated append of (key, id) for the lanes with `in` set; keeps s.c (all
// matches), s.kmin / s.kmax; entries past `cap` are counted, not stored.
__device__ __forceinline__ void append(bool in, uint32_t key, int id, uint32_t* ok, int32_t* oi,
                                       int cap) {
  Smem& s = sm();
  const int lane = threadIdx.x & 31;
  const uint32_t bal = __ballot_sync(0xffffffffu, in);
  if (bal == 0u) return;
  const int leader = __ffs(bal) - 1;
  int slot0 = 0;
  if (lane == leader) slot0 = atomicAdd(&s.c, __popc(bal));
  slot0 = __shfl_sync(0xffffffffu, slot0, leader);
  if (in) {
    const int slot = slot0 + __popc(bal & ((1u << lane) - 1u));
    if (slot < cap) { ok[slot] = key; oi[slot] = id; }
    const uint32_t lo = __reduce_min_sync(bal, key), hi = __reduce_max_sync(bal, key);
    if (lane == leader) { atomicMin(&s.kmin, lo); atomicMax(&s.kmax, hi); }
  }
}

__device__ __forceinline__ void compact_begin() {
  Smem& s = sm();
  if (threadIdx.x == 0) { s.c = 0; s.kmin = 0xffffffffu; s.kmax = 0u; }
  __syncthreads();
}

// ---------------------------------------------------------------- passes over the row
// The row's blocks matched by p appended contiguously to the list (rare paths).
__device__ __noinline__ void compact_row(int N, Pred p) {
  Smem& s = sm();
  const float* x = row_x();
  compact_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = warp * 32; base < N; base += NT) {
    const int i = base + lane;
    float v = 0.f;
    uint32_t key = 0u;
    bool in = false;
    if (i < N) { v = x[i]; key = order_key(v); in = pred_in(p, v, key); }
    append(in, key, i, s.lk, s.li, DN_LIST);
  }
  __syncthreads();
}

__device__ __noinline__ void hist_row(int N, Pred p, float ml2) {
  Smem& s = sm();
  const float* x = row_x();
  const int tid = threadIdx.x;
#pragma unroll
  for (int b = 0; b < DN_BINS; ++b) s.hist[b * NT + tid] = 0.f;
  for (int i = tid; i < N; i += NT) {
    const float v = x[i];
    const uint32_t key = order_key(v);
    if (key >= p.ka && key <= p.kb) s.hist[bin_key(key, p.kb, p.mul) * NT + tid] += mass(v, ml2);
  }
  __syncthreads();
}

// Ties: of the c blocks with key tk, the number m whose mass first reaches T from acc.
__device__ __forceinline__ int tie_count(uint32_t tk, int c, double acc, double T, float ml2) {
  const double et = mass(key_value(tk), ml2);
  double need = et > 0.0 ? ceil((T - acc) / et) : static_cast<double>(c);
  if (!(need >= 1.0)) need = 1.0;
  if (need > static_cast<double>(c)) need = static_cast<double>(c);
  return static_cast<int>(need);
}

// The last kept block is the m-th block of the row with key tk in id order.
__device__ __noinline__ void tie_row(int N, int NW, uint32_t tk, int m) {
  Smem& s = sm();
  const float* x = row_x();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* words = reinterpret_cast<uint32_t*>(s.hist);  // NW <= DN_BINS * NT words
  for (int q = warp; q < NW; q += NWARP) {
    const int i = q * 32 + lane;
    const uint32_t b = __ballot_sync(0xffffffffu, i < N && order_key(x[i]) == tk);
    if (lane == 0) words[q] = b;
  }
  __syncthreads();
  if (tid == 0) {
    s.tau_key = tk;
    s.tau_id = 0x7fffffff;
    int seen = 0;
    for (int q = 0; q < NW; ++q) {
      const uint32_t b = words[q];
      const int n = __popc(b);
      if (seen + n >= m) {
        uint32_t bb = b;
        for (int k = seen + 1; k < m; ++k) bb &= bb - 1u;
        s.tau_id = q * 32 + __ffs(bb) - 1;
        break;
      }
      seen += n;
    }
  }
}

struct RowSplit {
  double acc;
  int done;
};

// Bin j0 holds more blocks than a list segment: compact it contiguously, and while it
// exceeds the list split it by key, until its blocks fit (done = 0, the list holds them)
// or share one logit (done = 1, tau fixed).
__device__ __noinline__ RowSplit refine_row(const DenoiseArgs& a, float M, float ml2, double T,
                                            double acc, int j0) {
  Smem& s = sm();
  const int N = a.N;
  compact_row(N, Pred{true, M, 0u, 0xffffffffu, 0ull, j0});
  int c = s.c;
  uint32_t kmin = s.kmin, kmax = s.kmax;
  for (int it = 0; c > DN_LIST; ++it) {
    if (kmin == kmax) {
      tie_row(N, a.NW, kmin, tie_count(kmin, c, acc, T, ml2));
      return RowSplit{acc, 1};
    }
    if (it == DN_MAX_REFINE) {  // unreachable: each split shrinks the key range 16-fold
      if (threadIdx.x == 0) {
        s.tau_key = kmax;
        s.tau_id = 0x7fffffff;
        set_err(a.err, LSA_DEVERR_NUMERIC);
      }
      return RowSplit{acc, 1};
    }
    Pred q = key_split(M, kmin, kmax);
    __syncthreads();  // every thread has read s.c, s.kmin, s.kmax and s.bsum
    hist_row(N, q, ml2);
    reduce_bins();
    q.jsel = choose_bin(T, acc);
    compact_row(N, q);
    c = s.c;
    kmin = s.kmin;
    kmax = s.kmax;
  }
  return RowSplit{acc, 0};
}

// ---------------------------------------------------------------- the candidate list
// Slot j = tid + NT*u (u < DN_SLOTS) of this thread is valid when bit u is set.
__device__ __forceinline__ uint32_t list_slots() {
  const Smem& s = sm();
  uint32_t v = 0u;
#pragma unroll
  for (int u = 0; u < DN_SLOTS; ++u) {
    const int j = threadIdx.x + NT * u;
    if ((j % DN_SEG) < s.cw[j / DN_SEG]) v |= 1u << u;
  }
  return v;
}

// The list entries matched by p, into s.ckey / s.cid (s.c, s.kmin, s.kmax as for rows).
__device__ __noinline__ void compact_list(uint32_t slots, Pred p) {
  Smem& s = sm();
  compact_begin();
#pragma unroll
  for (int u = 0; u < DN_SLOTS; ++u) {
    const int j = threadIdx.x + NT * u;
    uint32_t key = 0u;
    int id = 0;
    bool in = false;
    if ((slots >> u) & 1u) {
      key = s.lk[j];
      id = s.li[j];
      in = pred_in(p, key_value(key), key);
    }
    append(in, key, id, s.ckey, s.cid, DN_CAND);
  }
  __syncthreads();
}

__device__ __noinline__ void hist_list(uint32_t slots, Pred p, float ml2) {
  Smem& s = sm();
  float* col = s.hist + threadIdx.x;
#pragma unroll
  for (int b = 0; b < DN_BINS; ++b) col[b * NT] = 0.f;
#pragma unroll
  for (int u = 0; u < DN_SLOTS; ++u) {
    if (!((slots >> u) & 1u)) continue;
    const uint32_t key = s.lk[threadIdx.x + NT * u];
    if (key >= p.ka && key <= p.kb) col[bin_key(key, p.kb, p.mul) * NT] += mass(key_value(key), ml2);
  }
  __syncthreads();
}

// Ranks candidates s.ckey/s.cid[0..c) (c >= 1) by (key desc, id asc), scans their mass
// in rank order from acc and sets s.tau_key / s.tau_id to the first rank reaching T
// (the last rank when none does).
__device__ __noinline__ void rank_pick(int c, double acc, double T, float ml2) {
  Smem& s = sm();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // G adjacent lanes share one candidate's comparisons (G a power of two, G * c <= NT)
  int G = 32;
  while (G > 1 && G * c > NT) G >>= 1;
  const int i = tid / G, part = tid % G;
  uint32_t ki = 0u;
  int ii = 0, r = 0;
  if (i < c) {
    ki = s.ckey[i];
    ii = s.cid[i];
    for (int j = part; j < c; j += G) {
      const uint32_t kj = s.ckey[j];
      r += (kj > ki) | ((kj == ki) & (s.cid[j] < ii));
    }
  }
  for (int o = G / 2; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  if (i < c && part == 0) {
    s.se[r] = static_cast<double>(mass(key_value(ki), ml2));
    s.spos[r] = i;
  }
  if (tid == 0) s.pick = c - 1;
  __syncthreads();
  double v = tid < c ? s.se[tid] : 0.0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) s.wsum[warp] = v;
  __syncthreads();
  double before = acc;
  for (int k = 0; k < warp; ++k) before += s.wsum[k];
  if (tid < c && before + v >= T) atomicMin(&s.pick, tid);
  __syncthreads();
  if (tid == 0) {
    const int slot = s.spos[s.pick];
    s.tau_key = s.ckey[slot];
    s.tau_id = s.cid[slot];
  }
}

// The list (every block of one bin of the row) narrowed by key splits to at most
// DN_CAND candidates, which are ranked; fixes s.tau_key / s.tau_id.
__device__ __noinline__ void resolve_list(const DenoiseArgs& a, float M, float ml2, double T,
                                          double acc) {
  Smem& s = sm();
  const int tid = threadIdx.x;
  const uint32_t slots = list_slots();
  // all entries into the candidate arrays (when they fit), with their key range
  Pred q{false, M, 0u, 0xffffffffu, 0ull, -1};
  compact_list(slots, q);
  int c = s.c;
  uint32_t kmin = s.kmin, kmax = s.kmax;
  for (int it = 0;; ++it) {
    if (c == 0) {  // only for non-finite logits: the chosen bin always holds mass
      if (tid == 0) { s.tau_key = 0xffffffffu; s.tau_id = -1; set_err(a.err, LSA_DEVERR_NUMERIC); }
      return;
    }
    if (c <= DN_CAND) {
      rank_pick(c, acc, T, ml2);
      return;
    }
    if (kmin == kmax) {  // every block of the row with this logit is in the list
      tie_row(a.N, a.NW, kmin, tie_count(kmin, c, acc, T, ml2));
      return;
    }
    if (it == DN_MAX_REFINE) {
      if (tid == 0) { s.tau_key = kmax; s.tau_id = 0x7fffffff; set_err(a.err, LSA_DEVERR_NUMERIC); }
      return;
    }
    q = key_split(M, kmin, kmax);
    __syncthreads();  // every thread has read s.c, s.kmin, s.kmax and s.bsum
    hist_list(slots, q, ml2);
    reduce_bins();
    q.jsel = choose_bin(T, acc);
    compact_list(slots, q);
    c = s.c;
    kmin = s.kmin;
    kmax = s.kmax;
  }
}

// ---------------------------------------------------------------- the window's vote
// Run by the window's last CTA: bit-sliced counters over the L mask words of each
// 32-block group, labels written as a mask and as increasing ids. `lab` is shared
// scratch of NW words.
__device__ __noinline__ void vote_window(const DenoiseArgs& a, int w, uint32_t* lab) {
  Smem& s = sm();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NW = a.NW, L = a.L, vmin = a.min_votes;
  for (int q = tid; q < NW; q += NT) {
    uint32_t pl[DN_PLANES];
#pragma unroll
    for (int b = 0; b < DN_PLANES; ++b) pl[b] = 0u;
    const uint32_t* col = a.set_mask + static_cast<size_t>(w) * L * NW + q;
    for (int l0 = 0; l0 < L; l0 += 8) {
      uint32_t wv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        wv[u] = l0 + u < L ? __ldcg(col + static_cast<size_t>(l0 + u) * NW) : 0u;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t carry = wv[u];
#pragma unroll
        for (int b = 0; b < DN_PLANES; ++b) {
          const uint32_t t = pl[b] & carry;
          pl[b] ^= carry;
          carry = t;
        }
      }
    }
    uint32_t ge;
    if (vmin <= 0) {
      ge = 0xffffffffu;
    } else if (vmin >= (1 << DN_PLANES)) {
      ge = 0u;
    } else {
      uint32_t gt = 0u, eq = 0xffffffffu;  // count > vmin, count == vmin so far
#pragma unroll
      for (int b = DN_PLANES - 1; b >= 0; --b) {
        if ((vmin >> b) & 1) {
          eq &= pl[b];
        } else {
          gt |= eq & pl[b];
          eq &= ~pl[b];
        }
      }
      ge = gt | eq;
    }
    const int valid = a.N - q * 32;
    if (valid < 32) ge &= (1u << valid) - 1u;
    lab[q] = ge;
    if (a.label_mask) a.label_mask[static_cast<size_t>(w) * NW + q] = ge;
  }
  __syncthreads();
  // ordered compaction: thread t owns words [t * per, (t + 1) * per)
  const int per = (NW + NT - 1) / NT;
  const int q0 = tid * per, q1 = min(NW, q0 + per);
  int cnt = 0;
  for (int q = q0; q < q1; ++q) cnt += __popc(lab[q]);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) s.wcnt[warp] = incl;
  __syncthreads();
  int pos = incl - cnt;
  for (int k = 0; k < warp; ++k) pos += s.wcnt[k];
  if (tid == NT - 1) s.total = pos + cnt;
  int32_t* ids = a.label_ids + static_cast<size_t>(w) * a.label_cap;
  for (int q = q0; q < q1 && pos < a.label_cap; ++q) {
    uint32_t b = lab[q];
    while (b != 0u && pos < a.label_cap) {
      ids[pos++] = q * 32 + __ffs(b) - 1;
      b &= b - 1u;
    }
  }
  __syncthreads();
  if (tid == 0) {
    a.label_cnt[w] = s.total;
    a.tickets[w] = 0u;  // ready for the next call
  }
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(NT, 2) denoise_kernel(const __grid_constant__ DenoiseArgs a) {
  Smem& s = sm();
  const int N = a.N, NW = a.NW;
  float* x = row_x();
  uint32_t* words = row_words(NW);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int w = row / a.L;
  const float* src = a.logits + static_cast<size_t>(row) * N;

  // ---- the row into shared memory; the row max
  float m = -INFINITY;
  if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(a.logits) & 15u) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* x4 = reinterpret_cast<float4*>(x);
#pragma unroll 8
    for (int i = tid; i < N / 4; i += NT) {
      const float4 v = __ldcs(s4 + i);
      x4[i] = v;
      m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
    }
  } else {
#pragma unroll 8
    for (int i = tid; i < N; i += NT) {
      const float v = __ldcs(src + i);
      x[i] = v;
      m = fmaxf(m, v);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s.wmax[warp] = m;
  __syncthreads();
  float M = s.wmax[0];
#pragma unroll
  for (int k = 1; k < NWARP; ++k) M = fmaxf(M, s.wmax[k]);
  const float ml2 = M * DN_LOG2E;

  // ---- pass 1: mass by whole units below the max
  {
    float* col = s.hist + tid;
#pragma unroll
    for (int b = 0; b < DN_BINS; ++b) col[b * NT] = 0.f;
#pragma unroll 8
    for (int i = tid; i < N; i += NT) {
      const float v = x[i];
      col[bin0(v, M) * NT] += mass(v, ml2);
    }
    __syncthreads();
  }
  reduce_bins();
  double S = 0.0;
  for (int j = 0; j < DN_BINS; ++j) S += s.bsum[j];
  const double T = a.top_p * S;
  double acc = 0.0;
  const int j0 = choose_bin(T, acc);

  // ---- pass 2: mask words of the blocks above bin j0; bin j0 into the warp's segment
  {
    uint32_t* sk = s.lk + warp * DN_SEG;
    int32_t* si = s.li + warp * DN_SEG;
    int off = 0;
#pragma unroll 4
    for (int q = warp; q < NW; q += NWARP) {
      const int i = q * 32 + lane;
      const float v = i < N ? x[i] : -INFINITY;
      const int jb = bin0(v, M);
      const uint32_t ab = __ballot_sync(0xffffffffu, i < N && jb < j0);
      if (lane == 0) words[q] = ab;
      const bool in = i < N && jb == j0;
      const uint32_t bb = __ballot_sync(0xffffffffu, in);
      if (bb != 0u) {
        if (in) {
          const int slot = off + __popc(bb & ((1u << lane) - 1u));
          if (slot < DN_SEG) { sk[slot] = order_key(v); si[slot] = i; }
        }
        off += __popc(bb);
      }
    }
    if (lane == 0) s.cw[warp] = off;
    __syncthreads();
  }
  bool ovf = false;
#pragma unroll
  for (int k = 0; k < NWARP; ++k) ovf |= s.cw[k] > DN_SEG;

  // ---- rare: bin j0 overflowed a segment. Compact it contiguously (splitting it over
  // the row while it exceeds the list); the mask is then derived from the row.
  bool from_row = false;
  int done = 0;
  if (ovf) {
    __syncthreads();  // every thread has read cw
    const RowSplit rs = refine_row(a, M, ml2, T, acc, j0);
    acc = rs.acc;
    done = rs.done;
    from_row = true;
    __syncthreads();
    if (tid < NWARP) {  // the contiguous list seen as segments
      const int c = min(s.c, DN_LIST);
      s.cw[tid] = max(0, min(DN_SEG, c - tid * DN_SEG));
    }
    __syncthreads();
  }
  if (!done) resolve_list(a, M, ml2, T, acc);
  __syncthreads();

  const uint32_t tk = s.tau_key;
  const int ti = s.tau_id;
  if (!from_row) {
    // ---- the kept list entries OR-ed into the words of the blocks above the bin
    const uint32_t slots = list_slots();
#pragma unroll
    for (int u = 0; u < DN_SLOTS; ++u) {
      if (!((slots >> u) & 1u)) continue;
      const int j = tid + NT * u;
      const uint32_t key = s.lk[j];
      const int id = s.li[j];
      if (key > tk || (key == tk && id <= ti)) atomicOr(&words[id >> 5], 1u << (id & 31));
    }
  } else {
    // ---- the mask from the row
    for (int q = warp; q < NW; q += NWARP) {
      const int i = q * 32 + lane;
      bool sel = false;
      if (i < N) {
        const uint32_t key = order_key(x[i]);
        sel = key > tk || (key == tk && i <= ti);
      }
      const uint32_t b = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) words[q] = b;
    }
  }
  __syncthreads();
  int cnt = 0;
  uint32_t* out = a.set_mask + static_cast<size_t>(row) * NW;
  for (int q = tid; q < NW; q += NT) {
    const uint32_t b = words[q];
    out[q] = b;
    cnt += __popc(b);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);

  // ---- the row's set size, the window ticket, the vote when this row closes the window
  if (lane == 0) s.wcnt[warp] = cnt;
  __threadfence();  // the mask words before the window's ticket
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int k = 0; k < NWARP; ++k) t += s.wcnt[k];
    if (a.set_cnt) a.set_cnt[row] = t;
    __threadfence();
    s.last = atomicAdd(&a.tickets[w], 1u) == static_cast<uint32_t>(a.L - 1);
  }
  __syncthreads();
  if (!s.last) return;
  __threadfence();
  vote_window(a, w, words);
}

size_t smem_bytes(int32_t NW) {
  return sizeof(Smem) + static_cast<size_t>(NW) * 32 * sizeof(float) +
         static_cast<size_t>(NW) * sizeof(uint32_t);
}

static_assert(LSA_DENOISE_MAX_BLOCKS % 32 == 0, "whole mask words");
static_assert(sizeof(Smem) + LSA_DENOISE_MAX_BLOCKS * 4 + LSA_DENOISE_MAX_BLOCKS / 8 <= 227 * 1024,
              "the longest row fits one CTA's shared memory");
static_assert(LSA_DENOISE_MAX_BLOCKS / 32 <= DN_BINS * NT, "tie words fit the histogram area");
static_assert(DN_CAND <= NT, "one scan lane per ranked candidate");

}  // namespace
}  // namespace lsa

extern "C" size_t lsa_denoise_workspace_size(int32_t n_windows) {
  if (n_windows <= 0) return 0;
  return (static_cast<size_t>(n_windows) * sizeof(uint32_t) + 255u) / 256u * 256u;
}

extern "C" lsa_status lsa_denoise_labels(const float* logits, int32_t n_windows,
                                         int32_t n_layers, int32_t n_blocks, double top_p,
                                         int32_t min_votes, uint32_t* set_mask,
                                         int32_t* set_cnt, uint32_t* label_mask,
                                         int32_t* label_ids, int32_t label_cap,
                                         int32_t* label_cnt, void* ws, size_t ws_bytes,
                                         int32_t* err, void* stream) {
  using namespace lsa;
  if (logits == nullptr || set_mask == nullptr || label_cnt == nullptr || ws == nullptr)
    return LSA_ERR_INVALID_ARG;
  if (n_windows < 1 || n_layers < 1 || n_layers >= (1 << DN_PLANES) || n_blocks < 1 ||
      n_blocks > LSA_DENOISE_MAX_BLOCKS)
    return LSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(n_windows) * n_layers > 0x7fffffffLL) return LSA_ERR_INVALID_ARG;
  if (!(top_p > 0.0) || !(top_p <= 1.0)) return LSA_ERR_INVALID_ARG;
  if (label_cap < 0 || (label_cap > 0 && label_ids == nullptr)) return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 3u) != 0 ||
      ws_bytes < lsa_denoise_workspace_size(n_windows))
    return LSA_ERR_INVALID_ARG;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(denoise_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes(LSA_DENOISE_MAX_BLOCKS / 32))) !=
        cudaSuccess)
      return LSA_ERR_CUDA;
    attr = true;
  }
  DenoiseArgs a{};
  a.logits = logits;
  a.W = n_windows;
  a.L = n_layers;
  a.N = n_blocks;
  a.NW = (n_blocks + 31) / 32;
  a.top_p = top_p;
  a.min_votes = min_votes;
  a.set_mask = set_mask;
  a.set_cnt = set_cnt;
  a.label_mask = label_mask;
  a.label_ids = label_ids;
  a.label_cap = label_cap;
  a.label_cnt = label_cnt;
  a.tickets = static_cast<uint32_t*>(ws);
  a.err = err;
  denoise_kernel<<<n_windows * n_layers, NT, smem_bytes(a.NW), static_cast<cudaStream_t>(stream)>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
