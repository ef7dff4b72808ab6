// Label denoising of the indexer's training targets ("FlashMemory-DeepSeek-V4 Explained",
// zhichai.net, section 3 "Label Denoising Pipeline"): for every token window and every
// CSA layer, a softmax over the layer's raw Lightning-Indexer logits of all KV blocks;
// the smallest set of blocks whose probabilities reach top_p (0.6 on the page); then a
// block is a label of the window when at least min_votes (3 of the 21) layers kept it.
//
// Persistent CTAs, two per SM, each taking rows (window, layer) in turn. A row sits in
// shared memory. Once the row's last read is done, one bulk copy brings the CTA's next
// row in, and it lands while the current row is being finished. Each thread owns whole
// 32-block mask words and reads its word's 32 logits as eight 16-byte loads. The loads
// start at a lane-dependent chunk, so that a warp's loads hit every bank once. The top-p
// set is found without sorting the row:
//   1. row max M, then e_i = 2^(x_i*log2(e) - M*log2(e)) for every block. A 16-bin
//      histogram of the mass by whole logit units d_i = M - x_i gives the total S and
//      the bin j0 where the running mass from the top crosses T = top_p * S;
//   2. one pass writes each word's blocks above bin j0 (kept whatever the boundary) and
//      its blocks in bin j0. It also adds each block of bin j0 to a 256-way split of the
//      bin, linear in d: a count and an exact 64-bit fixed-point mass per part, by
//      32-bit shared atomics;
//   3. the part where the running mass crosses T is chosen. Only the blocks of bin j0
//      are visited again: those in earlier parts join the mask, and those in the chosen
//      part become the candidate list (their number is known from step 2);
//   4. one warp ranks up to 32 candidates by (logit descending, id ascending) and scans
//      their mass in that order in fp64. The candidates up to the first rank whose
//      running mass reaches T join the mask. A longer list is first split 256 ways by the
//      order-preserving integer key of the logit, the same way, until at most 32
//      candidates remain. When more than 32 remain and all share one logit, the first m
//      of them by id are kept, m the smallest count whose mass reaches T.
// When the chosen part holds more blocks than the list, it is first split 16 ways over
// the row, by key. Ordering uses the exact fp32 logits, so blocks with equal
// probability are the blocks with equal logits, and they are taken by increasing id. Only
// the position of the boundary depends on rounding: fp32 e_i, fp64 and fixed-point sums.
//
// In the first pass each thread accumulates its share of the histogram in its own
// shared-memory column (bank = lane), so the columns see no contention and each sums its
// blocks in a fixed order; the bins are summed in fp64. The vote is a second launch, one
// CTA per window, with saturating (or, for more than 8 votes, bit-sliced) counters over
// the layers' 32-block mask words.
#include "lsa_common.cuh"

#include <algorithm>
#include <atomic>
#include <mutex>

namespace lsa {
namespace {

constexpr int NT = 512;               // threads per CTA
constexpr int NWARP = NT / 32;
constexpr int DN_BINS = 16;           // first pass: whole logit units below the max
constexpr int DN_FINE = 256;          // splits of a bin or of a list
constexpr int DN_RANK = 32;           // candidates ranked by one warp
constexpr int DN_LIST = 2048;         // entries per list buffer
constexpr int DN_INBIN = 4096;        // ids of the blocks of bin j0, listed when they fit
constexpr int DN_MAX_REFINE = 8;      // 256-way key splits: 4 always suffice for 32-bit keys
constexpr int DN_MAX_SPLIT = 12;      // 16-way row splits: 8 always suffice
constexpr int DN_PLANES = 6;          // vote counter bit planes: counts up to 63 layers
constexpr float DN_LOG2E = 1.4426950408889634f;
// Split parts sum their blocks' mass in units of 2^-36 (a mass is at most 1, the row
// maximum's): 45,056 blocks sum below 2^52, exact in a double.
constexpr float FIX_SCALE = 68719476736.0f;        // 2^36
constexpr double FIX_UNIT = 1.0 / 68719476736.0;   // 2^-36

struct DenoiseArgs {
  const float* logits;   // [W][L][N]
  int32_t W, L, N, NW;   // NW = ceil(N / 32)
  int32_t rows;          // W * L
  int32_t bulk;          // rows are 16-byte aligned whole multiples of 16 bytes
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

// Shared memory: this fixed part, then the row (NW * 32 floats; the slots past N hold
// -inf), the mask words (NW) and the words of the blocks in bin j0 (NW). The first
// pass's per-thread histogram columns and, after them, the two candidate list buffers
// share the area `u`.
struct __align__(16) Smem {
  float u[DN_BINS * NT];     // hist columns | bin j0's ids [DN_INBIN] or keys1, ids1; keys0, ids0
  uint32_t flo[DN_FINE];              // split parts: mass in units of 2^-36, low half
  uint32_t fhi[DN_FINE];              // and high half
  uint32_t fcnt[DN_FINE];             // and block count
  double bsum[DN_BINS];
  uint64_t bar;              // the row copy's mbarrier
  float wmax[NWARP];
  int32_t wcnt[NWARP];
  uint32_t wkmin[NWARP], wkmax[NWARP];
  int32_t cnt[2];            // entries appended to each list buffer
  int32_t nin;               // blocks of bin j0 (their ids listed while they fit)
  int32_t pad_;
  int32_t jsel;              // chosen bin or part (choose, choose_fine)
  int32_t csel;              // blocks in the chosen part (choose_fine)
  int32_t tau_id;            // mth_marked
  int32_t abort;             // a bounded wait gave up
  double acc;                // mass above the chosen bin or part
  double total_mass;         // all bins' mass
  double T;                  // top_p times the row's mass
};

extern __shared__ __align__(16) unsigned char dn_smem[];
__device__ __forceinline__ Smem& sm() { return *reinterpret_cast<Smem*>(dn_smem); }
// List buffer 0 takes the second half of u, buffer 1 the first half, which holds the ids
// of bin j0's blocks until the candidates are listed.
__device__ __forceinline__ uint32_t* list_k(int b) {
  return reinterpret_cast<uint32_t*>(sm().u) + (1 - b) * 2 * DN_LIST;
}
__device__ __forceinline__ int32_t* list_i(int b) {
  return reinterpret_cast<int32_t*>(sm().u) + (1 - b) * 2 * DN_LIST + DN_LIST;
}
__device__ __forceinline__ int32_t* inbin_ids() { return reinterpret_cast<int32_t*>(sm().u); }
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

// The first pass bins blocks by whole logit units below R = ceil(M), an integer at or
// above every logit of the row: bin(x) = min(floor(R - x), 15). A sum in [2^23, 2^24)
// rounded toward -inf is 2^23 plus the floor of the exact sum, so the float's bits minus
// those of 2^23 give the floor. With |R| <= 2^22, R + 2^23 is exact, and one add of -x
// rounded down gives floor(R - x) exactly (EXACT). Otherwise the difference is rounded
// first, and every comparison below uses that rounded difference instead.
struct RowRef {
  float M, ml2;  // the row max and M * log2(e)
  float R;       // ceil(M)
  float RB;      // R + 2^23
};
template <bool EXACT>
__device__ __forceinline__ uint32_t floor_bits(const RowRef& r, float x) {
  return __float_as_uint(EXACT ? __fadd_rd(r.RB, -x) : __fadd_rd(r.R - x, 8388608.0f));
}
// min(floor, 15) from floor_bits; beyond 2^23 (and +inf, NaN) the block takes the last
// bin.
__device__ __forceinline__ int bin_of_bits(uint32_t bits) {
  // unsigned: bits below those of 2^23 (a negative or tiny sum, which x <= R rules out)
  // wrap around and take the last bin too
  return static_cast<int>(min(bits - 0x4b000000u, static_cast<uint32_t>(DN_BINS - 1)));
}

// Whether x lies above bin j0 (up) and above its lower edge (gt): EXACT compares x with
// the integers R - j0 and R - j0 - 1 (no rounding), the other form compares the rounded
// difference with j0 and j0 + 1. The last bin has no lower edge (finite x only).
struct Edges {
  float A, B;    // EXACT: up = x > A, gt = x > B
  float lo, hi;  // otherwise: up = R - x < lo, gt = R - x < hi
};
template <bool EXACT>
__device__ __forceinline__ void edges(const RowRef& r, float x, const Edges& e, bool& up, bool& gt) {
  if (EXACT) {
    up = x > e.A;
    gt = x > e.B;
  } else {
    const float d = r.R - x;
    up = d < e.lo;
    gt = d < e.hi;
  }
}

// The part of bin j0 that one of its blocks falls in, from d = R - x rounded: 256 parts
// of width 1/256 for a unit bin, of width 1/16 from 15 on for the last (unbounded) bin,
// the last part taking the rest. Non-decreasing in d, so parts are intervals of the logit.
__device__ __forceinline__ int fine_part(const RowRef& r, float x, float lo, bool last_bin) {
  const float t = ((r.R - x) - lo) * (last_bin ? 16.0f : 256.0f);
  return t < 255.0f ? static_cast<int>(fmaxf(t, 0.0f)) : DN_FINE - 1;
}

// NB linear bins of the key range [ka, kb], bin 0 holding the largest keys.
struct KeySplit {
  uint32_t ka, kb;
  uint64_t mul;  // floor(NB * 2^32 / (kb - ka + 1))
};
template <int NB>
__device__ __forceinline__ KeySplit key_split(uint32_t ka, uint32_t kb) {
  const uint64_t R = static_cast<uint64_t>(kb - ka) + 1ull;
  return KeySplit{ka, kb, (static_cast<uint64_t>(NB) << 32) / R};
}
template <int NB>
__device__ __forceinline__ int bin_key(const KeySplit& k, uint32_t key) {
  // below NB for every key in [ka, kb]; the clamp only bounds the index for other keys
  return min(static_cast<int>((static_cast<uint64_t>(k.kb - key) * k.mul) >> 32), NB - 1);
}

// Sets block id's bit in a word array of NW words; an id outside the row (which no valid
// list holds) is skipped and reported.
__device__ __forceinline__ void mark(uint32_t* words, int NW, int32_t id, int32_t* err) {
  if (id >= 0 && (id >> 5) < NW)
    atomicOr(&words[id >> 5], 1u << (id & 31));
  else
    set_err(err, LSA_DEVERR_BAD_SIZE);
}

// Appends (key, id) to list buffer b when there is room (the count always advances).
__device__ __forceinline__ void push(int b, uint32_t key, int32_t id) {
  const int pos = atomicAdd(&sm().cnt[b], 1);
  if (pos < DN_LIST) {
    list_k(b)[pos] = key;
    list_i(b)[pos] = id;
  }
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Appends the lanes with `take` set to list buffer b: one shared atomic per warp, the
// lanes in lane order after it. Called by all 32 lanes of a warp.
__device__ __forceinline__ void append(int b, bool take, uint32_t key, int32_t id) {
  const uint32_t w = __ballot_sync(0xffffffffu, take);
  if (w == 0u) return;
  int base = 0;
  if ((threadIdx.x & 31) == __ffs(w) - 1) base = atomicAdd(&sm().cnt[b], __popc(w));
  base = __shfl_sync(0xffffffffu, base, __ffs(w) - 1);
  const int pos = base + __popc(w & lanemask_lt());
  if (take && pos < DN_LIST) {
    list_k(b)[pos] = key;
    list_i(b)[pos] = id;
  }
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

__device__ __forceinline__ void choose_fine_warp(double T, double acc);

// The answer of a choice over bins or parts: the chosen one, its block count (parts
// only), the mass above it and the threshold T.
struct Pick {
  int j;
  int cnt;
  double acc;
  double T;
};

// Scans 16 bins in s.bsum from the top for the first non-empty bin where acc + the
// running mass reaches T (the last non-empty bin when rounding leaves the total short
// of T). With top_p > 0, T is top_p times the bins' total. Every warp computes the same
// answer from 16 values, so no barrier follows; thread 0 also leaves it in s.
__device__ __forceinline__ Pick choose(double T, double acc, double top_p = 0.0) {
  Smem& s = sm();
  const int lane = threadIdx.x & 31;
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
  if (threadIdx.x == 0) {
    s.jsel = j;
    s.acc = acc + above;
    s.total_mass = total;
    s.T = T;
  }
  return Pick{j, 0, acc + above, T};
}

// The same choice over the 256 split parts in s.flo, s.fhi / s.fcnt (part 0 the largest
// logits): the first part holding blocks where acc + the running mass reaches T, else
// the last part holding blocks. The test runs on the exact fixed-point sums: the running
// sum must reach need = ceil((T - acc) * 2^36). Lane l scans parts 8l .. 8l + 7 after a
// scan of the lanes' sums. Warp 0 computes; every thread has the answer after the
// barrier.
__device__ __forceinline__ Pick choose_fine(double T, double acc) {
  Smem& s = sm();
  if (threadIdx.x < 32) choose_fine_warp(T, acc);
  __syncthreads();
  return Pick{s.jsel, s.csel, s.acc, T};
}

// choose_fine() for the lanes of warp 0; lane 0 leaves the answer in s.
__device__ __forceinline__ void choose_fine_warp(double T, double acc) {
  Smem& s = sm();
  const int lane = threadIdx.x & 31;
  unsigned long long f[8];
  {
    const uint4* lo = reinterpret_cast<const uint4*>(s.flo + lane * 8);
    const uint4* hi = reinterpret_cast<const uint4*>(s.fhi + lane * 8);
    const uint4 l0 = lo[0], l1 = lo[1], h0 = hi[0], h1 = hi[1];
    f[0] = (static_cast<unsigned long long>(h0.x) << 32) | l0.x;
    f[1] = (static_cast<unsigned long long>(h0.y) << 32) | l0.y;
    f[2] = (static_cast<unsigned long long>(h0.z) << 32) | l0.z;
    f[3] = (static_cast<unsigned long long>(h0.w) << 32) | l0.w;
    f[4] = (static_cast<unsigned long long>(h1.x) << 32) | l1.x;
    f[5] = (static_cast<unsigned long long>(h1.y) << 32) | l1.y;
    f[6] = (static_cast<unsigned long long>(h1.z) << 32) | l1.z;
    f[7] = (static_cast<unsigned long long>(h1.w) << 32) | l1.w;
  }
  uint32_t n[8];
  const uint4* csrc = reinterpret_cast<const uint4*>(s.fcnt + lane * 8);
  const uint4 c0 = csrc[0], c1 = csrc[1];
  n[0] = c0.x; n[1] = c0.y; n[2] = c0.z; n[3] = c0.w;
  n[4] = c1.x; n[5] = c1.y; n[6] = c1.z; n[7] = c1.w;
  unsigned long long mine = 0ull;
#pragma unroll
  for (int k = 0; k < 8; ++k) mine += f[k];
  unsigned long long incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  const double nd = (T - acc) * 68719476736.0;
  const unsigned long long need =
      !(nd > 0.0) ? 0ull : (nd < 1.8e19 ? static_cast<unsigned long long>(ceil(nd)) : ~0ull);
  unsigned long long run = incl - mine, above_hit = 0ull, above_last = 0ull;
  int hit = -1, last = -1;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    if (n[k] != 0u) {
      if (hit < 0 && run + f[k] >= need) {
        hit = k;
        above_hit = run;
      }
      last = k;
      above_last = run;
    }
    run += f[k];
  }
  const uint32_t hb = __ballot_sync(0xffffffffu, hit >= 0);
  const uint32_t nb = __ballot_sync(0xffffffffu, last >= 0);
  const int src_lane = hb ? __ffs(hb) - 1 : (nb ? 31 - __clz(nb) : 0);
  const int k = max(__shfl_sync(0xffffffffu, hb ? hit : last, src_lane), 0);
  const unsigned long long above = __shfl_sync(0xffffffffu, hb ? above_hit : above_last, src_lane);
  uint32_t cnt = 0u;
#pragma unroll
  for (int t = 0; t < 8; ++t) cnt = t == k ? n[t] : cnt;
  cnt = __shfl_sync(0xffffffffu, cnt, src_lane);
  if (lane == 0) {
    s.jsel = src_lane * 8 + k;
    s.csel = static_cast<int>(cnt);
    s.acc = acc + static_cast<double>(above) * FIX_UNIT;
  }
}

// Adds one block to a split part: its count, and its mass in fixed point as an exact
// 64-bit sum kept in two 32-bit words. The low word's add returns the old value, which
// shows whether it wrapped; the high word then takes the mass's high half plus that carry.
// However the adds interleave, high * 2^32 + low ends as the exact sum. (32-bit shared
// atomics: a 64-bit atomic add in their place made the whole call 8 % slower.)
__device__ __forceinline__ void fine_add(int part, float e) {
  Smem& s = sm();
  atomicAdd(&s.fcnt[part], 1u);
  const unsigned long long v = __float2ull_rz(e * FIX_SCALE);
  const uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
  const uint32_t old = atomicAdd(&s.flo[part], lo);
  const uint32_t carry = old + lo < old ? 1u : 0u;
  if (hi + carry != 0u) atomicAdd(&s.fhi[part], hi + carry);
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

// The tied blocks marked in bin_words: the first m of them by id join the mask words.
__device__ __noinline__ void keep_first_marked(int NW, int m) {
  mth_marked(NW, m);
  const int ti = sm().tau_id;
  uint32_t* mw = mask_words(NW);
  const uint32_t* bw = bin_words(NW);
  for (int q = threadIdx.x; q < NW; q += NT) {
    const int first = q * 32;
    uint32_t b = bw[q];
    if (first > ti) b = 0u;
    else if (first + 31 > ti) b &= (2u << (ti - first)) - 1u;
    mw[q] |= b;
  }
  __syncthreads();
}

// One warp ranks the c (0..32) entries of list buffer b by (key desc, id asc), scans their
// mass in rank order from acc, and ORs the entries up to the first rank whose running
// mass reaches T (all of them when none does) into the mask words.
__device__ __noinline__ void rank_warp(int NW, int b, int c, double acc, double T, float ml2,
                                       int32_t* err) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const bool v = lane < c;
    const uint32_t ki = v ? list_k(b)[lane] : 0u;
    const int ii = v ? list_i(b)[lane] : 0x7fffffff;
    const double e = v ? static_cast<double>(mass(key_value(ki), ml2)) : 0.0;
    int r = 0;
    double before = 0.0;  // mass of the entries ranked before this one
#pragma unroll 4
    for (int j = 0; j < c; ++j) {
      const uint32_t kj = __shfl_sync(0xffffffffu, ki, j);
      const int ij = __shfl_sync(0xffffffffu, ii, j);
      const double ej = __shfl_sync(0xffffffffu, e, j);
      const bool ahead = (kj > ki) | ((kj == ki) & (ij < ii));
      r += ahead;
      before += ahead ? ej : 0.0;
    }
    const bool hit = v && acc + before + e >= T;
    const int rmin = __reduce_min_sync(0xffffffffu, hit ? r : 0x7fffffff);
    const int want = rmin == 0x7fffffff ? c - 1 : rmin;
    if (v && r <= want) mark(mask_words(NW), NW, ii, err);
    if (lane == 0 && c == 0) set_err(err, LSA_DEVERR_NUMERIC);  // only non-finite logits
  }
  __syncthreads();
}

// The candidate list (buffer 0, s.cnt[0] <= DN_LIST entries, any order) narrowed by
// 256-way key splits to at most DN_RANK entries, then ranked; entries split off above the
// chosen part join the mask words. All c entries equal: the first m by id are kept.
__device__ __noinline__ void resolve_list(const DenoiseArgs& a, float ml2, double T, double acc) {
  Smem& s = sm();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NW = a.NW;
  uint32_t* mw = mask_words(NW);
  int b = 0;
  for (int it = 0;; ++it) {
    const int c = min(s.cnt[b], DN_LIST);
    if (c <= DN_RANK) {
      rank_warp(NW, b, c, acc, T, ml2, a.err);
      return;
    }
    const uint32_t* lk = list_k(b);
    const int32_t* li = list_i(b);
    if (it == DN_MAX_REFINE) {  // unreachable: each split shrinks the key range 256-fold
      if (tid == 0) set_err(a.err, LSA_DEVERR_NUMERIC);
      __syncthreads();
      return;
    }
    // the entries' key range; clear the split parts
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int j = tid; j < c; j += NT) {
      const uint32_t k = lk[j];
      lo = min(lo, k);
      hi = max(hi, k);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) { s.wkmin[warp] = lo; s.wkmax[warp] = hi; }
    if (tid < DN_FINE) { s.flo[tid] = 0u; s.fhi[tid] = 0u; s.fcnt[tid] = 0u; }
    __syncthreads();
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) {
      kmin = min(kmin, s.wkmin[w]);
      kmax = max(kmax, s.wkmax[w]);
    }
    if (kmin == kmax) {  // all tied: mark them, keep the first m by id
      uint32_t* bw = bin_words(NW);
      for (int q = tid; q < NW; q += NT) bw[q] = 0u;
      __syncthreads();
      for (int j = tid; j < c; j += NT) mark(bw, NW, li[j], a.err);
      __syncthreads();
      keep_first_marked(NW, tie_count(kmin, c, acc, T, ml2));
      return;
    }
    const KeySplit ks = key_split<DN_FINE>(kmin, kmax);
    for (int j = tid; j < c; j += NT) {
      const uint32_t k = lk[j];
      fine_add(bin_key<DN_FINE>(ks, k), mass(key_value(k), ml2));
    }
    if (tid == 0) s.cnt[b ^ 1] = 0;  // last read at this round's start, before a barrier
    __syncthreads();
    const Pick pf = choose_fine(T, acc);
    const int jsel = pf.j;
    acc = pf.acc;
    // above the chosen part: into the mask; the chosen part: into the other buffer
    for (int j0 = 0; j0 < c; j0 += NT) {  // whole warps take every round (ballots)
      const int j = j0 + tid;
      uint32_t k = 0u;
      int32_t id = 0;
      int part = DN_FINE;
      if (j < c) {
        k = lk[j];
        id = li[j];
        part = bin_key<DN_FINE>(ks, k);
        if (part < jsel) mark(mw, NW, id, a.err);
      }
      append(b ^ 1, part == jsel, k, id);
    }
    __syncthreads();
    b ^= 1;
  }
}

// Rare: the chosen part holds more than DN_LIST blocks (c of them, keys in [kmin, kmax]:
// a part is an interval of the logit, so its blocks are exactly the row's blocks with
// keys in that range). Splits it 16 ways by key over the row, the blocks above the
// chosen split joining the mask words, until the part fits the list (then it becomes list
// buffer 0) or shares one logit (then its first m blocks by id are kept). Returns 1 in
// the second case. s.acc holds the mass above the part on return.
__device__ __noinline__ int split_row(const DenoiseArgs& a, float ml2, double T, int c,
                                      uint32_t kmin, uint32_t kmax) {
  Smem& s = sm();
  const int N = a.N, NW = a.NW;
  const float* x = row_x();
  uint32_t* mw = mask_words(NW);
  uint32_t* bw = bin_words(NW);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double acc = s.acc;
  for (int it = 0;; ++it) {
    if (c <= DN_LIST) {  // the part becomes the list
      if (tid == 0) s.cnt[0] = 0;
      __syncthreads();
      for (int q = warp; q < NW; q += NWARP) {
        const int i = q * 32 + lane;
        const uint32_t k = i < N ? order_key(x[i]) : 0u;
        append(0, i < N && k >= kmin && k <= kmax, k, i);
      }
      __syncthreads();
      return 0;
    }
    if (kmin == kmax) {  // ties over the row
      for (int q = warp; q < NW; q += NWARP) {
        const int i = q * 32 + lane;
        const uint32_t t = __ballot_sync(0xffffffffu, i < N && order_key(x[i]) == kmin);
        if (lane == 0) bw[q] = t;
      }
      __syncthreads();
      keep_first_marked(NW, tie_count(kmin, c, acc, T, ml2));
      return 1;
    }
    if (it == DN_MAX_SPLIT) {  // unreachable: each split shrinks the key range 16-fold
      if (tid == 0) set_err(a.err, LSA_DEVERR_NUMERIC);
      __syncthreads();
      return 1;
    }
    const KeySplit ks = key_split<DN_BINS>(kmin, kmax);
    float* col = s.u + tid;
#pragma unroll
    for (int k = 0; k < DN_BINS; ++k) col[k * NT] = 0.f;
    for (int i = tid; i < N; i += NT) {
      const uint32_t key = order_key(x[i]);
      if (key >= kmin && key <= kmax) col[bin_key<DN_BINS>(ks, key) * NT] += mass(x[i], ml2);
    }
    __syncthreads();
    reduce_columns();
    const Pick ps = choose(T, acc);
    const int jsel = ps.j;
    acc = ps.acc;
    int n = 0;
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int q = warp; q < NW; q += NWARP) {
      const int i = q * 32 + lane;
      const uint32_t key = i < N ? order_key(x[i]) : 0u;
      const bool in_range = i < N && key >= kmin && key <= kmax;
      const int bin = in_range ? bin_key<DN_BINS>(ks, key) : DN_BINS;
      const uint32_t up = __ballot_sync(0xffffffffu, bin < jsel);
      if (lane == 0) mw[q] |= up;
      if (bin == jsel) {
        ++n;
        lo = min(lo, key);
        hi = max(hi, key);
      }
    }
    block_scan(n, &c, lo, hi, &kmin, &kmax);  // starts with a barrier: the mask words are done
  }
}
// ---------------------------------------------------------------- the window's vote
// The blocks of one 32-block group kept by at least V (1..8) of the window's L layers:
// saturating counters, ge[j] holding the blocks seen in at least j + 1 layers so far.
// col points at the group's word of layer 0; the layers are NW words apart.
template <int V>
__device__ __forceinline__ uint32_t at_least(const uint32_t* col, int L, int NW) {
  uint32_t ge[V];
#pragma unroll
  for (int j = 0; j < V; ++j) ge[j] = 0u;
  for (int l0 = 0; l0 < L; l0 += 16) {  // 16 loads in flight at once
    uint32_t wv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u)
      wv[u] = l0 + u < L ? __ldcg(col + static_cast<size_t>(l0 + u) * NW) : 0u;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
#pragma unroll
      for (int j = V - 1; j > 0; --j) ge[j] |= ge[j - 1] & wv[u];
      ge[0] |= wv[u];
    }
  }
  return ge[V - 1];
}

// Any threshold: bit-sliced counters of the layer count (DN_PLANES planes), then the
// blocks whose count is at least vmin.
__device__ __forceinline__ uint32_t at_least_any(const uint32_t* col, int L, int NW, int vmin) {
  if (vmin >= (1 << DN_PLANES)) return 0u;
  uint32_t pl[DN_PLANES];
#pragma unroll
  for (int b = 0; b < DN_PLANES; ++b) pl[b] = 0u;
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
  return gt | eq;
}

// The labels of window w (blocks kept by at least min_votes of its layers), written as a
// mask and as increasing ids. `lab` is shared scratch of NW words.
__device__ __noinline__ void vote_window(const DenoiseArgs& a, int w, uint32_t* lab) {
  const int tid = threadIdx.x;
  const int NW = a.NW, L = a.L, vmin = a.min_votes;
  for (int q = tid; q < NW; q += NT) {
    const uint32_t* col = a.set_mask + static_cast<size_t>(w) * L * NW + q;
    uint32_t ge;
    switch (vmin) {
      case 1: ge = at_least<1>(col, L, NW); break;
      case 2: ge = at_least<2>(col, L, NW); break;
      case 3: ge = at_least<3>(col, L, NW); break;
      case 4: ge = at_least<4>(col, L, NW); break;
      case 5: ge = at_least<5>(col, L, NW); break;
      case 6: ge = at_least<6>(col, L, NW); break;
      case 7: ge = at_least<7>(col, L, NW); break;
      case 8: ge = at_least<8>(col, L, NW); break;
      default: ge = vmin <= 0 ? 0xffffffffu : at_least_any(col, L, NW, vmin); break;
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
}

// ---------------------------------------------------------------- the kernel
// Thread 0: one bulk copy of row r into the row buffer, completing on s.bar.
__device__ __forceinline__ void issue_row(const DenoiseArgs& a, int r) {
  Smem& s = sm();
  const uint32_t bytes = static_cast<uint32_t>(a.N) * 4u;
  mbar_arrive_expect_tx(&s.bar, bytes);
  bulk_load(row_x(), a.logits + static_cast<size_t>(r) * a.N, bytes, &s.bar);
}

// Pass 1 over one word: each block's mass into this thread's column of its bin.
template <bool EXACT>
__device__ __forceinline__ void hist_word(const float4* w4, int rot, const RowRef& r, float* col) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 v = w4[(k + rot) & 7];
    const float xs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) col[bin_of_bits(floor_bits<EXACT>(r, xs[c])) * NT] += mass(xs[c], r.ml2);
  }
}

// Pass 2 over one word: the bits of its blocks above bin j0 (up) and above the bin's
// lower edge (gt), in block order.
template <bool EXACT>
__device__ __forceinline__ void edge_word(const float4* w4, int rot, const RowRef& r, const Edges& e,
                                          uint32_t& up, uint32_t& gt) {
  up = 0u;
  gt = 0u;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 v = w4[(k + rot) & 7];
    const float xs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      bool u, g;
      edges<EXACT>(r, xs[c], e, u, g);
      up |= static_cast<uint32_t>(u) << (4 * k + c);
      gt |= static_cast<uint32_t>(g) << (4 * k + c);
    }
  }
  // chunk (k + rot) & 7 went to bits 4k .. 4k + 3: rotate into block order
  up = __funnelshift_l(up, up, 4 * rot);
  gt = __funnelshift_l(gt, gt, 4 * rot);
}

__global__ void __launch_bounds__(NT, 2) denoise_kernel(const __grid_constant__ DenoiseArgs a) {
  Smem& s = sm();
  const int N = a.N, NW = a.NW;
  float* x = row_x();
  const float4* x4 = reinterpret_cast<const float4*>(x);
  uint32_t* mw = mask_words(NW);
  uint32_t* bw = bin_words(NW);
  const int tid = threadIdx.x, lane = tid & 31;
  // a thread reads chunk (k + rot) & 7 of its word at step k: 8 lanes cover all banks
  const int rot = lane & 7;
  const bool bulk = a.bulk != 0;
  // the slots past N (never written by a row copy) hold -inf: no mass, never above the
  // boundary, never in bin j0
  for (int i = N + tid; i < NW * 32; i += NT) x[i] = -INFINITY;
  if (tid == 0) {
    s.abort = 0;
    mbar_init(&s.bar, 1);
    fence_barrier_init();  // the initialised barrier is visible to the copy engine
  }
  __syncthreads();
  if (bulk && tid == 0 && static_cast<int>(blockIdx.x) < a.rows) issue_row(a, blockIdx.x);
  grid_dependents_launch();  // the vote kernel may be scheduled as SMs free up
  uint32_t parity = 0u;
  for (int row = blockIdx.x; row < a.rows; row += gridDim.x) {
    // ---- the row in shared memory; the row max
    bool failed = false;
    if (bulk) {
      failed = !mbar_wait(&s.bar, parity, &s.abort);
      parity ^= 1u;
    } else {
      const float* src = a.logits + static_cast<size_t>(row) * N;
#pragma unroll 8
      for (int i = tid; i < N; i += NT) x[i] = __ldcs(src + i);
      __syncthreads();
    }
    float m = -INFINITY;
    if (!failed) {
      for (int q = tid; q < NW; q += NT) {
        const float4* w4 = x4 + q * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 v = w4[(k + rot) & 7];
          m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s.wmax[tid >> 5] = m;
    if (tid == 0) {  // this row's lists
      s.cnt[0] = 0;
      s.nin = 0;
    }
    if (tid < DN_FINE) {         // this row's split of bin j0
      s.flo[tid] = 0u;
      s.fhi[tid] = 0u;
      s.fcnt[tid] = 0u;
    }
    if (__syncthreads_or(failed)) {
      if (tid == 0) {
        set_err(a.err, LSA_DEVERR_TIMEOUT);
        mbar_wait(&s.bar, parity ^ 1u, nullptr);  // the copy in flight, once more (bounded)
      }
      return;
    }
    RowRef ref;
    ref.M = s.wmax[0];
#pragma unroll
    for (int k = 1; k < NWARP; ++k) ref.M = fmaxf(ref.M, s.wmax[k]);
    ref.ml2 = ref.M * DN_LOG2E;
    ref.R = ceilf(ref.M);
    ref.RB = ref.R + 8388608.0f;
    const bool exact = fabsf(ref.R) <= 4194304.0f;

    // ---- pass 1: mass by whole units below R, in this thread's column
    {
      float* col = s.u + tid;
#pragma unroll
      for (int k = 0; k < DN_BINS; ++k) col[k * NT] = 0.f;
      for (int q = tid; q < NW; q += NT) {
        if (exact) hist_word<true>(x4 + q * 8, rot, ref, col);
        else hist_word<false>(x4 + q * 8, rot, ref, col);
      }
      __syncthreads();
    }
    reduce_columns();
    const Pick p0 = choose(0.0, 0.0, a.top_p);  // T = top_p * S with the row's total S
    const double T = p0.T;
    double acc = p0.acc;
    const int j0 = p0.j;

    // ---- pass 2: per word, the blocks above bin j0 and those in it; bin j0's blocks
    // into its 256-way split
    const bool last_bin = j0 == DN_BINS - 1;
    Edges e;
    e.lo = static_cast<float>(j0);
    e.hi = last_bin ? INFINITY : e.lo + 1.0f;
    e.A = ref.R - e.lo;
    e.B = last_bin ? -INFINITY : e.A - 1.0f;
    // the loop runs the same rounds in every lane (warp-wide appends)
    for (int q0 = 0; q0 < NW; q0 += NT) {
      const int q = q0 + tid;
      uint32_t up = 0u, gt = 0u;
      if (q < NW) {
        if (exact) edge_word<true>(x4 + q * 8, rot, ref, e, up, gt);
        else edge_word<false>(x4 + q * 8, rot, ref, e, up, gt);
      }
      const uint32_t in = gt & ~up;
      if (q < NW) {
        mw[q] = up;
        bw[q] = in;
      }
      // bin j0's ids into the list: one shared atomic per warp
      const int n = __popc(in);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const int total = __shfl_sync(0xffffffffu, incl, 31);
      int base = 0;
      if (lane == 31 && total > 0) base = atomicAdd(&s.nin, total);
      base = __shfl_sync(0xffffffffu, base, 31);
      int pos = base + incl - n;
      // bin j0's blocks into its 256-way split: the warp's listed blocks spread over its
      // lanes; a warp whose blocks did not fit the list takes them word by word
      if (base + total <= DN_INBIN) {
        int32_t* ids = inbin_ids();
        for (uint32_t b = in; b != 0u; b &= b - 1u) ids[pos++] = q * 32 + __ffs(b) - 1;
        __syncwarp();
        for (int j = lane; j < total; j += 32) {
          const float v = x[ids[base + j]];
          fine_add(fine_part(ref, v, e.lo, last_bin), mass(v, ref.ml2));
        }
      } else {
        for (uint32_t b = in; b != 0u; b &= b - 1u) {
          const float v = x[q * 32 + __ffs(b) - 1];
          fine_add(fine_part(ref, v, e.lo, last_bin), mass(v, ref.ml2));
        }
      }
    }
    __syncthreads();
    const int nin = s.nin;
    const bool listed = nin <= DN_INBIN;
    const Pick pf = choose_fine(T, acc);
    const int fsel = pf.j;
    const int c = pf.cnt;
    acc = pf.acc;

    // ---- pass 3: bin j0's blocks again: earlier parts into the mask, the chosen part
    // into the candidate list (when it fits) and its key range
    {
      const bool list_it = c <= DN_LIST;
      uint32_t klo = 0xffffffffu, khi = 0u;
      if (listed) {
        const int32_t* ids = inbin_ids();
        for (int j = tid; j < nin; j += NT) {
          const int id = ids[j];
          const float v = x[id];
          const int f = fine_part(ref, v, e.lo, last_bin);
          if (f < fsel) {
            mark(mw, NW, id, a.err);
          } else if (f == fsel) {
            const uint32_t key = order_key(v);
            klo = min(klo, key);
            khi = max(khi, key);
            if (list_it) push(0, key, id);
          }
        }
      } else {
        for (int q = tid; q < NW; q += NT) {
          uint32_t up = 0u;
          for (uint32_t b = bw[q]; b != 0u; b &= b - 1u) {
            const int p = __ffs(b) - 1;
            const float v = x[q * 32 + p];
            const int f = fine_part(ref, v, e.lo, last_bin);
            if (f < fsel) {
              up |= 1u << p;
            } else if (f == fsel) {
              const uint32_t key = order_key(v);
              klo = min(klo, key);
              khi = max(khi, key);
              if (list_it) push(0, key, q * 32 + p);
            }
          }
          if (up != 0u) atomicOr(&mw[q], up);
        }
      }
      int fixed = 0;
      if (list_it) {
        __syncthreads();
      } else {
        int dummy;
        uint32_t kmin, kmax;
        block_scan(0, &dummy, klo, khi, &kmin, &kmax);
        fixed = split_row(a, ref.ml2, T, c, kmin, kmax);
        acc = s.acc;
      }
      // the row buffer is free: the CTA's next row is copied in while this one finishes
      if (bulk && tid == 0 && row + static_cast<int>(gridDim.x) < a.rows)
        issue_row(a, row + gridDim.x);
      if (!fixed) resolve_list(a, ref.ml2, T, acc);
    }

    // ---- the row's mask words and set size
    int cnt = 0;
    uint32_t* out = a.set_mask + static_cast<size_t>(row) * NW;
    for (int q = tid; q < NW; q += NT) {
      const uint32_t b = mw[q];
      out[q] = b;
      cnt += __popc(b);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (lane == 0) s.wcnt[tid >> 5] = cnt;
    __syncthreads();
    if (tid == 0 && a.set_cnt) {
      int t = 0;
      for (int k = 0; k < NWARP; ++k) t += s.wcnt[k];
      a.set_cnt[row] = t;
    }
  }
}

// The vote, one CTA per window, launched after denoise_kernel on the same stream as a
// programmatic dependent: its CTAs take the SMs that the last rows free, then wait until
// every set mask is written. Shared memory is Smem, then NW words of scratch.
__global__ void __launch_bounds__(NT, 1) vote_kernel(const __grid_constant__ DenoiseArgs a) {
  grid_dependency_wait();
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
static_assert(4 * DN_LIST * 4 <= sizeof(float) * DN_BINS * NT, "both lists fit the shared area");
static_assert(DN_INBIN <= 2 * DN_LIST, "bin j0's ids fit list buffer 1's place");
static_assert(LSA_DENOISE_MAX_BLOCKS % 32 == 0, "whole mask words");
static_assert(sizeof(Smem) + LSA_DENOISE_MAX_BLOCKS * 4 + LSA_DENOISE_MAX_BLOCKS / 4 <= 227 * 1024,
              "the longest row fits one CTA's shared memory");
static_assert(LSA_DENOISE_MAX_BLOCKS * 4 < (1 << 20), "a row copy fits an mbarrier's count");
static_assert(LSA_DENOISE_MAX_BLOCKS * 68719476736.0 < 9007199254740992.0,
              "a split part's fixed-point mass is exact in a double");

// Resident row-kernel CTAs per SM for `smem` bytes of dynamic shared memory on the current
// device (the occupancy query, cached per device and size: it is host work per call
// otherwise). 0 on error.
int ctas_per_sm(size_t smem) {
  struct Entry {
    int dev;
    size_t smem;
    int per_sm;
  };
  static std::mutex mu;
  static Entry done[64];
  static int n_done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].dev == dev && done[i].smem == smem) return done[i].per_sm;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, denoise_kernel, NT, smem) !=
      cudaSuccess)
    return 0;
  if (n_done < 64) done[n_done++] = Entry{dev, smem, per_sm};
  return per_sm;
}

// Launches kern<<<grid, NT, smem, st>>>(a) as a programmatic dependent of the stream's
// preceding work, or plainly where the device refuses that (remembered per device).
lsa_status launch_pdl(dim3 grid, size_t smem, cudaStream_t st,
                      void (*kern)(const DenoiseArgs), const DenoiseArgs& a, int dev) {
  static std::atomic<int> pdl_refused[64];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_refused[dev].load(std::memory_order_relaxed) ? 0 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
  if (e == cudaErrorNotSupported && cfg.numAttrs == 1) {
    cudaGetLastError();
    pdl_refused[dev].store(1, std::memory_order_relaxed);
    cfg.numAttrs = 0;
    e = cudaLaunchKernelEx(&cfg, kern, a);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

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
  a.rows = n_windows * n_layers;
  a.bulk = ((n_blocks & 3) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0) ? 1 : 0;
  a.top_p = top_p;
  a.min_votes = min_votes;
  a.set_mask = set_mask;
  a.set_cnt = set_cnt;
  a.label_mask = label_mask;
  a.label_ids = label_ids;
  a.label_cap = label_cap;
  a.label_cnt = label_cnt;
  a.err = err;
  // persistent: as many CTAs as fit at once, each taking every grid-th row
  const size_t smem = smem_bytes(a.NW);
  int dev = 0;
  const int sms = lsa_host::sm_count();
  const int per_sm = ctas_per_sm(smem);
  if (cudaGetDevice(&dev) != cudaSuccess || sms < 1 || per_sm < 1) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  const int grid = static_cast<int>(std::min<int64_t>(a.rows, static_cast<int64_t>(per_sm) * sms));
  // the vote as a programmatic dependent of the row kernel (measured: the row kernel
  // itself is faster launched plainly, its CTAs then pair up on the SMs as they should)
  if (dev < 0 || dev >= 64) return LSA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  denoise_kernel<<<grid, NT, smem, st>>>(a);
  lsa_status r = cudaPeekAtLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
  if (r == LSA_OK) r = launch_pdl(dim3(n_windows), vote_smem_bytes(a.NW), st, vote_kernel, a, dev);
  return r;
}
