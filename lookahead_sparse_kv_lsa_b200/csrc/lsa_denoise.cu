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
//   2. one pass of warp ballots writes, per 32 blocks, the mask word of the blocks above
//      bin j0 (kept whatever the boundary) and the word of the blocks in bin j0;
//   3. the blocks of bin j0 become a candidate list in increasing id (one block-wide
//      scan over the words); the list is split 16 ways, linearly in the
//      order-preserving integer key of the logit, and narrowed in place, the entries
//      above the chosen part OR-ed into the mask, until at most 256 candidates remain;
//   4. those are ranked by (logit descending, id ascending), their mass is scanned in
//      that order in fp64, and the first rank whose running mass reaches T fixes the
//      last kept (logit, id); the kept candidates are OR-ed into the mask. When all the
//      remaining candidates share one logit, the first m of them by id are kept, m the
//      smallest count whose mass reaches T.
// When bin j0 holds more blocks than the list, the bin is split the same way over the
// row first. Ordering uses the exact fp32 logits, so blocks with equal probability are
// the blocks with equal logits and they are taken by increasing id; only the position of
// the boundary depends on rounding (fp32 e_i, fp64 sums).
//
// In the first pass each thread accumulates its share of the histogram in its own
// shared-memory column (bank = lane), so the mass needs no shared atomics; the bins are
// summed in fp64. The vote is a second launch, one CTA per window, as bit-sliced counters
// over the layers' 32-block mask words.
#include "lsa_common.cuh"

namespace lsa {
namespace {

constexpr int NT = 512;               // threads per CTA
constexpr int NWARP = NT / 32;
constexpr int DN_BINS = 16;
constexpr int DN_CAND = 256;          // candidates resolved by ranking
constexpr int DN_MAX_REFINE = 12;     // key-range splits; 9 always suffice for 32-bit keys
constexpr int DN_PLANES = 6;          // vote counter bit planes: counts up to 63 layers
constexpr int DN_LIST = 2048;         // candidate list
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
  int32_t* err;
};

// Shared memory: this fixed part, then the row (NW * 32 floats), the mask words (NW) and
// the words of the blocks in the bin being resolved (NW). The first pass's per-thread
// histogram columns and, after it, the candidate list share the area `u`.
struct __align__(16) Smem {
  float u[DN_BINS * NT];     // hist columns | list keys [DN_LIST], list ids [DN_LIST]
  double bsum[DN_BINS];
  double wsum[NWARP];
  double se[DN_CAND];        // candidate mass in rank order
  int32_t spos[DN_CAND];     // rank -> list position
  float lhist[NWARP][DN_BINS];  // list split: per-warp bin mass
  float wmax[NWARP];
  int32_t wcnt[NWARP];
  uint32_t wkmin[NWARP], wkmax[NWARP];
  int32_t c;                 // list entries
  uint32_t kmin, kmax;       // their key range
  int32_t pick;              // rank of the last kept candidate
  uint32_t tau_key;          // the last kept (key, id)
  int32_t tau_id;
  int32_t jsel;              // chosen bin (choose)
  int32_t last;              // this CTA closes its window
  int32_t total;
  double acc;                // mass above the chosen bin
  double total_mass;         // all bins' mass
  double T;                  // top_p times the row's mass
};

extern __shared__ __align__(16) unsigned char dn_smem[];
__device__ __forceinline__ Smem& sm() { return *reinterpret_cast<Smem*>(dn_smem); }
__device__ __forceinline__ uint32_t* list_k() { return reinterpret_cast<uint32_t*>(sm().u); }
__device__ __forceinline__ int32_t* list_i() { return reinterpret_cast<int32_t*>(sm().u) + DN_LIST; }
__device__ __forceinline__ float* row_x() { return reinterpret_cast<float*>(dn_smem + sizeof(Smem)); }
__device__ __forceinline__ uint32_t* mask_words(int NW) {
  return reinterpret_cast<uint32_t*>(row_x() + static_cast<size_t>(NW) * 32);
}
__device__ __forceinline__ uint32_t* bin_words(int NW) { return mask_words(NW) + NW; }

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

__device__ __forceinline__ int bin0(float v, float M) {
  return max(0, min(static_cast<int>(M - v), DN_BINS - 1));  // M - v >= 0 when finite
}

// 16 linear bins of the key range [ka, kb], bin 0 holding the largest keys.
struct KeySplit {
  uint32_t ka, kb;
  uint64_t mul;  // floor(16 * 2^32 / (kb - ka + 1))
};
__device__ __forceinline__ KeySplit key_split(uint32_t ka, uint32_t kb) {
  const uint64_t R = static_cast<uint64_t>(kb - ka) + 1ull;
  return KeySplit{ka, kb, (static_cast<uint64_t>(DN_BINS) << 32) / R};
}
__device__ __forceinline__ int bin_key(const KeySplit& k, uint32_t key) {
  return static_cast<int>((static_cast<uint64_t>(k.kb - key) * k.mul) >> 32);
}

// Block-wide exclusive scan of one int per thread; *total gets the sum, *klo / *khi the
// min / max of the threads' key ranges lo / hi. Uses s.wcnt, s.wkmin, s.wkmax.
__device__ __forceinline__ int block_scan(int v, int* total, uint32_t lo = 0xffffffffu,
                                          uint32_t hi = 0u, uint32_t* klo = nullptr,
                                          uint32_t* khi = nullptr) {
  Smem& s = sm();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  lo = __reduce_min_sync(0xffffffffu, lo);
  hi = __reduce_max_sync(0xffffffffu, hi);
  __syncthreads();  // the previous use has been read
  if (lane == 31) { s.wcnt[warp] = incl; s.wkmin[warp] = lo; s.wkmax[warp] = hi; }
  __syncthreads();
  int before = 0, all = 0;
  uint32_t l = 0xffffffffu, h = 0u;
#pragma unroll
  for (int k = 0; k < NWARP; ++k) {
    const int t = s.wcnt[k];
    before += k < warp ? t : 0;
    all += t;
    l = min(l, s.wkmin[k]);
    h = max(h, s.wkmax[k]);
  }
  *total = all;
  if (klo) *klo = l;
  if (khi) *khi = h;
  return before + incl - v;
}

// Scans 16 bins in s.bsum from the top for the first non-empty bin where acc + the
// running mass reaches T (the last non-empty bin when rounding leaves the total short
// of T): s.jsel is that bin, s.acc the mass above it, s.total_mass the sum of all bins.
// With top_p > 0, T is top_p times that sum (s.T). Warp 0 computes; every thread reads
// the answer after the barrier.
__device__ __forceinline__ void choose(double T, double acc, double top_p = 0.0) {
  Smem& s = sm();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const double bj = lane < DN_BINS ? s.bsum[lane] : 0.0;
    double incl = bj;  // running mass of bins 0..lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const double total = __shfl_sync(0xffffffffu, incl, DN_BINS - 1);
    if (top_p > 0.0) T = top_p * total;
    const uint32_t nz = __ballot_sync(0xffffffffu, bj > 0.0);
    const uint32_t hit = __ballot_sync(0xffffffffu, bj > 0.0 && acc + incl >= T);
    const int j = hit ? __ffs(hit) - 1 : (nz ? 31 - __clz(nz) : 0);
    const double above = __shfl_sync(0xffffffffu, incl - bj, j);
    if (lane == 0) {
      s.jsel = j;
      s.acc = acc + above;
      s.total_mass = total;
      s.T = T;
    }
  }
  __syncthreads();
}

// Sums the NT per-thread histogram columns into s.bsum (fp64; a warp per bin).
__device__ __forceinline__ void reduce_columns() {
  Smem& s = sm();
  static_assert(NT / DN_BINS == 32, "one warp per bin");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double v = 0.0;
#pragma unroll 4
  for (int k = 0; k < NT / 32; ++k) v += s.u[warp * NT + lane + 32 * k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) s.bsum[warp] = v;
  __syncthreads();
}

// The blocks marked in bin_words, in increasing id, into the list (the first DN_LIST of
// them): s.c = their number, s.kmin / s.kmax their key range.
__device__ __noinline__ void build_list(int NW) {
  Smem& s = sm();
  const float* x = row_x();
  const uint32_t* bw = bin_words(NW);
  const int tid = threadIdx.x;
  const int per = (NW + NT - 1) / NT;
  const int q0 = tid * per, q1 = min(NW, q0 + per);
  int cnt = 0;
  uint32_t lo = 0xffffffffu, hi = 0u;
  for (int q = q0; q < q1; ++q) {
    uint32_t b = bw[q];
    cnt += __popc(b);
    while (b != 0u) {
      const uint32_t key = order_key(x[q * 32 + __ffs(b) - 1]);
      b &= b - 1u;
      lo = min(lo, key);
      hi = max(hi, key);
    }
  }
  int total;
  uint32_t klo, khi;
  int pos = block_scan(cnt, &total, lo, hi, &klo, &khi);
  uint32_t* lk = list_k();
  int32_t* li = list_i();
  for (int q = q0; q < q1 && pos < DN_LIST; ++q) {
    uint32_t b = bw[q];
    while (b != 0u && pos < DN_LIST) {
      const int id = q * 32 + __ffs(b) - 1;
      b &= b - 1u;
      lk[pos] = order_key(x[id]);
      li[pos] = id;
      ++pos;
    }
  }
  if (tid == 0) { s.c = total; s.kmin = klo; s.kmax = khi; }
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

// The id of the m-th (1-based) block marked in bin_words, in increasing id, into
// s.tau_id (0x7fffffff when there are fewer).
__device__ __noinline__ void mth_marked(int NW, int m) {
  Smem& s = sm();
  const uint32_t* bw = bin_words(NW);
  const int tid = threadIdx.x;
  const int per = (NW + NT - 1) / NT;
  const int q0 = tid * per, q1 = min(NW, q0 + per);
  int cnt = 0;
  for (int q = q0; q < q1; ++q) cnt += __popc(bw[q]);
  int total;
  const int before = block_scan(cnt, &total);
  if (tid == 0) s.tau_id = 0x7fffffff;
  __syncthreads();
  if (m > before && m <= before + cnt) {
    int seen = before;
    for (int q = q0; q < q1; ++q) {
      const uint32_t b = bw[q];
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
  __syncthreads();
}

// Rare: bin j0 holds more than DN_LIST blocks. Split the marked blocks of the row by key
// (the blocks above the chosen part join the mask words) until the marked part fits the
// list or shares one logit. Returns 1 when tau is fixed (ties), 0 when the list holds
// the part; acc is updated.
__device__ __noinline__ int split_row(const DenoiseArgs& a, float ml2, double T, double* accp) {
  Smem& s = sm();
  const int N = a.N, NW = a.NW;
  const float* x = row_x();
  uint32_t* mw = mask_words(NW);
  uint32_t* bw = bin_words(NW);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double acc = *accp;
  for (int it = 0;; ++it) {
    const int c = s.c;
    const uint32_t kmin = s.kmin, kmax = s.kmax;
    if (c <= DN_LIST) { *accp = acc; return 0; }
    if (kmin == kmax) {
      mth_marked(NW, tie_count(kmin, c, acc, T, ml2));
      if (tid == 0) s.tau_key = kmin;
      __syncthreads();
      *accp = acc;
      return 1;
    }
    if (it == DN_MAX_REFINE) {  // unreachable: each split shrinks the key range 16-fold
      if (tid == 0) { s.tau_key = kmax; s.tau_id = 0x7fffffff; set_err(a.err, LSA_DEVERR_NUMERIC); }
      __syncthreads();
      *accp = acc;
      return 1;
    }
    const KeySplit ks = key_split(kmin, kmax);
    float* col = s.u + tid;
    __syncthreads();  // every thread has read s.c, s.kmin, s.kmax
#pragma unroll
    for (int b = 0; b < DN_BINS; ++b) col[b * NT] = 0.f;
    for (int i = tid; i < N; i += NT) {
      const uint32_t key = order_key(x[i]);
      if (key >= kmin && key <= kmax) col[bin_key(ks, key) * NT] += mass(x[i], ml2);
    }
    __syncthreads();
    reduce_columns();
    choose(T, acc);
    const int jsel = s.jsel;
    acc = s.acc;
    for (int q = warp; q < NW; q += NWARP) {
      const int i = q * 32 + lane;
      const uint32_t key = i < N ? order_key(x[i]) : 0u;
      const bool in_range = i < N && key >= kmin && key <= kmax;
      const int b = in_range ? bin_key(ks, key) : DN_BINS;
      const uint32_t up = __ballot_sync(0xffffffffu, b < jsel);
      const uint32_t in = __ballot_sync(0xffffffffu, b == jsel);
      if (lane == 0) { mw[q] |= up; bw[q] = in; }
    }
    __syncthreads();
    build_list(NW);
  }
}

// Ranks the list's first c (1..DN_CAND) entries by (key desc, id asc), scans their mass
// in rank order from acc and sets s.tau_key / s.tau_id to the first rank reaching T (the
// last rank when none does).
__device__ __noinline__ void rank_pick(int c, double acc, double T, float ml2) {
  Smem& s = sm();
  const uint32_t* lk = list_k();
  const int32_t* li = list_i();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (c <= 32) {  // one warp: lane j holds candidate j
    if (warp == 0) {
      const bool v = lane < c;
      const uint32_t ki = v ? lk[lane] : 0u;
      const int ii = v ? li[lane] : 0x7fffffff;
      const double e = v ? static_cast<double>(mass(key_value(ki), ml2)) : 0.0;
      int r = 0;
      double before = 0.0;  // mass of the candidates ranked before this one
      for (int j = 0; j < c; ++j) {
        const uint32_t kj = __shfl_sync(0xffffffffu, ki, j);
        const int ij = __shfl_sync(0xffffffffu, ii, j);
        const bool ahead = (kj > ki) | ((kj == ki) & (ij < ii));
        r += ahead;
        const double ej = __shfl_sync(0xffffffffu, e, j);
        if (ahead) before += ej;
      }
      const bool hit = v && acc + before + e >= T;
      const int rmin = __reduce_min_sync(0xffffffffu, hit ? r : 0x7fffffff);
      const int want = rmin == 0x7fffffff ? c - 1 : rmin;
      const uint32_t who = __ballot_sync(0xffffffffu, v && r == want);
      if (lane == __ffs(who) - 1) {
        s.tau_key = ki;
        s.tau_id = ii;
      }
    }
    __syncthreads();
    return;
  }
  // G adjacent lanes share one candidate's comparisons (G a power of two, G * c <= NT)
  int G = 32;
  while (G > 1 && G * c > NT) G >>= 1;
  const int i = tid / G, part = tid % G;
  uint32_t ki = 0u;
  int ii = 0, r = 0;
  if (i < c) {
    ki = lk[i];
    ii = li[i];
    for (int j = part; j < c; j += G) {
      const uint32_t kj = lk[j];
      r += (kj > ki) | ((kj == ki) & (li[j] < ii));
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
    s.tau_key = lk[slot];
    s.tau_id = li[slot];
  }
  __syncthreads();
}

// The list (c entries in increasing id) narrowed to at most DN_CAND candidates and
// resolved; the entries split off above the chosen part are OR-ed into the mask words.
// Fixes s.tau_key / s.tau_id.
__device__ __noinline__ void resolve_list(const DenoiseArgs& a, float ml2, double T, double acc) {
  Smem& s = sm();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* lk = list_k();
  int32_t* li = list_i();
  uint32_t* mw = mask_words(a.NW);
  for (int it = 0;; ++it) {
    const int c = s.c;
    const uint32_t kmin = s.kmin, kmax = s.kmax;
    if (c == 0) {  // only for non-finite logits: the chosen bin always holds mass
      if (tid == 0) { s.tau_key = 0xffffffffu; s.tau_id = -1; set_err(a.err, LSA_DEVERR_NUMERIC); }
      __syncthreads();
      return;
    }
    if (c <= DN_CAND) {
      rank_pick(c, acc, T, ml2);
      return;
    }
    if (kmin == kmax) {  // all tied and in increasing id: the m-th entry is the last kept
      if (tid == 0) {
        s.tau_key = kmin;
        s.tau_id = li[tie_count(kmin, c, acc, T, ml2) - 1];
      }
      __syncthreads();
      return;
    }
    if (it == DN_MAX_REFINE) {
      if (tid == 0) { s.tau_key = kmax; s.tau_id = 0x7fffffff; set_err(a.err, LSA_DEVERR_NUMERIC); }
      __syncthreads();
      return;
    }
    // split: per-warp bin mass by warp sums, one entry per thread per round
    const KeySplit ks = key_split(kmin, kmax);
    float part[DN_BINS];
#pragma unroll
    for (int b = 0; b < DN_BINS; ++b) part[b] = 0.f;
    for (int j0 = 0; j0 < c; j0 += NT) {
      const int j = j0 + tid;
      int b = -1;
      float e = 0.f;
      if (j < c) {
        const uint32_t key = lk[j];
        b = bin_key(ks, key);
        e = mass(key_value(key), ml2);
      }
#pragma unroll
      for (int k = 0; k < DN_BINS; ++k) {
        float t = b == k ? e : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        part[k] += t;
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < DN_BINS; ++k) s.lhist[warp][k] = part[k];
    }
    __syncthreads();
    if (tid < DN_BINS) {
      double v = 0.0;
      for (int w = 0; w < NWARP; ++w) v += s.lhist[w][tid];
      s.bsum[tid] = v;
    }
    __syncwarp();  // bins 0..15 are warp 0's lanes: choose() reads them in warp 0 only
    choose(T, acc);
    const int jsel = s.jsel;
    acc = s.acc;
    // entries above the chosen part join the mask; the chosen part is kept, in order
    uint32_t kk[DN_LIST / NT];
    int32_t ki[DN_LIST / NT];
    bool keep[DN_LIST / NT];
#pragma unroll
    for (int u = 0; u < DN_LIST / NT; ++u) {
      const int j = u * NT + tid;  // round u holds entries [u * NT, (u + 1) * NT)
      keep[u] = false;
      kk[u] = 0u;
      ki[u] = 0;
      if (j < c) {
        kk[u] = lk[j];
        ki[u] = li[j];
        const int b = bin_key(ks, kk[u]);
        if (b < jsel) atomicOr(&mw[ki[u] >> 5], 1u << (ki[u] & 31));
        keep[u] = b == jsel;
      }
    }
    // order-preserving compaction in place: every read above precedes the first write
    // (block_scan starts with a barrier); within a round the scan keeps thread order
    int base = 0;
    uint32_t klo = 0xffffffffu, khi = 0u;
#pragma unroll
    for (int u = 0; u < DN_LIST / NT; ++u) {
      if (u * NT >= c) break;  // uniform
      int tot_u;
      uint32_t l, h;
      const int pos = block_scan(keep[u] ? 1 : 0, &tot_u, keep[u] ? kk[u] : 0xffffffffu,
                                 keep[u] ? kk[u] : 0u, &l, &h);
      if (keep[u]) {
        lk[base + pos] = kk[u];
        li[base + pos] = ki[u];
      }
      base += tot_u;
      klo = min(klo, l);
      khi = max(khi, h);
    }
    if (tid == 0) { s.c = base; s.kmin = klo; s.kmax = khi; }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- the window's vote
// Bit-sliced counters over the L mask words of each 32-block group of window w, labels
// written as a mask and as increasing ids. `lab` is shared scratch of NW words.
__device__ __noinline__ void vote_window(const DenoiseArgs& a, int w, uint32_t* lab) {
  Smem& s = sm();
  const int tid = threadIdx.x;
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
  int total;
  int pos = block_scan(cnt, &total);
  int32_t* ids = a.label_ids + static_cast<size_t>(w) * a.label_cap;
  for (int q = q0; q < q1 && pos < a.label_cap; ++q) {
    uint32_t b = lab[q];
    while (b != 0u && pos < a.label_cap) {
      ids[pos++] = q * 32 + __ffs(b) - 1;
      b &= b - 1u;
    }
  }
  if (tid == 0) a.label_cnt[w] = total;
  (void)s;
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(NT, 2) denoise_kernel(const __grid_constant__ DenoiseArgs a) {
  Smem& s = sm();
  const int N = a.N, NW = a.NW;
  float* x = row_x();
  uint32_t* mw = mask_words(NW);
  uint32_t* bw = bin_words(NW);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
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
    float* col = s.u + tid;
#pragma unroll
    for (int b = 0; b < DN_BINS; ++b) col[b * NT] = 0.f;
#pragma unroll 8
    for (int i = tid; i < N; i += NT) {
      const float v = x[i];
      col[bin0(v, M) * NT] += mass(v, ml2);
    }
    __syncthreads();
  }
  reduce_columns();
  choose(0.0, 0.0, a.top_p);  // T = top_p * S with the row's total S
  const double T = s.T;
  double acc = s.acc;
  const int j0 = s.jsel;

  // ---- pass 2: per 32 blocks, the word of the blocks above bin j0 and of those in it.
  // bin0(v) < j0  <=>  M - v < j0;  bin0(v) == j0  <=>  j0 <= M - v < j0 + 1 (any
  // M - v from 15 on for the last bin), for finite logits.
  {
    const float lo = static_cast<float>(j0), hi = static_cast<float>(j0 + 1);
    const bool last_bin = j0 == DN_BINS - 1;
#pragma unroll 4
    for (int q = warp; q < NW; q += NWARP) {
      const int i = q * 32 + lane;
      const bool ok = i < N;
      const float d = M - (ok ? x[i] : 0.f);
      const uint32_t up = __ballot_sync(0xffffffffu, ok && d < lo);
      const uint32_t in = __ballot_sync(0xffffffffu, ok && d >= lo && (last_bin || d < hi));
      if (lane == 0) { mw[q] = up; bw[q] = in; }
    }
    __syncthreads();
  }

  // ---- the bin's blocks as a list (split over the row first when they overflow it)
  build_list(NW);
  int fixed = 0;
  if (s.c > DN_LIST) fixed = split_row(a, ml2, T, &acc);
  if (!fixed) resolve_list(a, ml2, T, acc);

  // ---- the kept candidates into the mask words
  const uint32_t tk = s.tau_key;
  const int ti = s.tau_id;
  {
    const int c = min(s.c, DN_LIST);
    const uint32_t* lk = list_k();
    const int32_t* li = list_i();
    if (!fixed) {
      for (int j = tid; j < c; j += NT) {
        const uint32_t key = lk[j];
        const int id = li[j];
        if (key > tk || (key == tk && id <= ti)) atomicOr(&mw[id >> 5], 1u << (id & 31));
      }
    } else {
      // ties over the row: the marked blocks with id up to tau_id
      for (int q = tid; q < NW; q += NT) {
        const int first = q * 32;
        uint32_t b = bw[q];
        if (first > ti) b = 0u;
        else if (first + 31 > ti) b &= (2u << (ti - first)) - 1u;
        mw[q] |= b;
      }
    }
    __syncthreads();
  }
  int cnt = 0;
  uint32_t* out = a.set_mask + static_cast<size_t>(row) * NW;
  for (int q = tid; q < NW; q += NT) {
    const uint32_t b = mw[q];
    out[q] = b;
    cnt += __popc(b);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);

  // ---- the row's set size
  if (lane == 0) s.wcnt[warp] = cnt;
  __syncthreads();
  if (tid == 0 && a.set_cnt) {
    int t = 0;
    for (int k = 0; k < NWARP; ++k) t += s.wcnt[k];
    a.set_cnt[row] = t;
  }
}

// The vote, one CTA per window, launched after denoise_kernel on the same stream (so all
// the window's set masks are complete): shared memory is Smem, then NW words of scratch.
__global__ void __launch_bounds__(NT, 1) vote_kernel(const __grid_constant__ DenoiseArgs a) {
  // no row here: the scratch words follow Smem directly (vote_smem_bytes)
  vote_window(a, blockIdx.x, reinterpret_cast<uint32_t*>(dn_smem + sizeof(Smem)));
}

size_t vote_smem_bytes(int32_t NW) {
  return sizeof(Smem) + static_cast<size_t>(NW) * sizeof(uint32_t);
}

size_t smem_bytes(int32_t NW) {
  return sizeof(Smem) + static_cast<size_t>(NW) * 32 * sizeof(float) +
         2 * static_cast<size_t>(NW) * sizeof(uint32_t);
}

static_assert(sizeof(Smem) % 16 == 0, "the row starts 16-byte aligned");
static_assert(2 * DN_LIST * 4 <= sizeof(float) * DN_BINS * NT, "the list fits the shared area");
static_assert(LSA_DENOISE_MAX_BLOCKS % 32 == 0, "whole mask words");
static_assert(sizeof(Smem) + LSA_DENOISE_MAX_BLOCKS * 4 + LSA_DENOISE_MAX_BLOCKS / 4 <= 227 * 1024,
              "the longest row fits one CTA's shared memory");
static_assert(DN_CAND <= NT, "one scan lane per ranked candidate");

}  // namespace
}  // namespace lsa

extern "C" lsa_status lsa_denoise_labels(const float* logits, int32_t n_windows,
                                         int32_t n_layers, int32_t n_blocks, double top_p,
                                         int32_t min_votes, uint32_t* set_mask,
                                         int32_t* set_cnt, uint32_t* label_mask,
                                         int32_t* label_ids, int32_t label_cap,
                                         int32_t* label_cnt, int32_t* err, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_denoise_labels");
  using namespace lsa;
  if (logits == nullptr || set_mask == nullptr || label_cnt == nullptr) return LSA_ERR_INVALID_ARG;
  if (n_windows < 1 || n_layers < 1 || n_layers >= (1 << DN_PLANES) || n_blocks < 1 ||
      n_blocks > LSA_DENOISE_MAX_BLOCKS)
    return LSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(n_windows) * n_layers > 0x7fffffffLL) return LSA_ERR_INVALID_ARG;
  if (!(top_p > 0.0) || !(top_p <= 1.0)) return LSA_ERR_INVALID_ARG;
  if (label_cap < 0 || (label_cap > 0 && label_ids == nullptr)) return LSA_ERR_INVALID_ARG;
  {
    lsa_status st = lsa_host::ensure_smem_limit(
        reinterpret_cast<const void*>(denoise_kernel),
        static_cast<int>(smem_bytes(LSA_DENOISE_MAX_BLOCKS / 32)));
    if (st == LSA_OK)
      st = lsa_host::ensure_smem_limit(reinterpret_cast<const void*>(vote_kernel),
                                       static_cast<int>(vote_smem_bytes(LSA_DENOISE_MAX_BLOCKS / 32)));
    if (st != LSA_OK) return st;
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
  a.err = err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  denoise_kernel<<<n_windows * n_layers, NT, smem_bytes(a.NW), st>>>(a);
  if (cudaPeekAtLastError() != cudaSuccess) return LSA_ERR_CUDA;
  vote_kernel<<<n_windows, NT, vote_smem_bytes(a.NW), st>>>(a);
  return cudaPeekAtLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
