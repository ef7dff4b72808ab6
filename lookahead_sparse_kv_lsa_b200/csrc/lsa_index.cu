// Neural Memory Indexer pass: query projection, block scoring, sign test, OR over the
// indexer layers, and ordered compaction of the kept block ids.
//
// "FlashMemory-DeepSeek-V4 Explained" (zhichai.net): section 2 steps 2-3 (score the
// historical blocks from the current hidden state, keep sigmoid > 0.5), section 3 (one
// small query projection per layer against frozen compressed block keys), section 4
// (independent indexers at three layers, OR-ed).
//
// One cooperative launch, one CTA per SM, three phases split by two grid barriers:
//
//  A. Warp 0 plans the CTA's share of K_idx rows and KW = 4 copy warps start their
//     16-byte asynchronous copies into shared memory (they do not depend on q); the
//     other warps compute the CTA's share of the W_q rows:
//     q[l][b][j] = W_q[l][j] . h[l][b] in fp32, each dot cut into four fixed parts
//     summed in a fixed order.
//  B. Scoring. The candidate rows of every sequence are grouped in 32-row "words"; all
//     words of the batch, in sequence order, are divided evenly over the CTAs. A warp
//     scores one word from shared memory, one lane per row (rows padded by 16 bytes so
//     the lanes' loads fall in different banks; the queries are broadcasts):
//     z_l = q_l . k / sqrt(d_i) + bias, keep bit z_l > 0 (equal to sigmoid(z_l) > 0.5);
//     one ballot per layer gives the word, OR-ed over the layers.
//  C. Compaction. Each CTA ranks the kept bits of its words (popcounts of the earlier
//     words of the same sequence, a warp scan over its own, kept in shared memory since
//     phase B) and writes the ascending id list; the CTA holding a sequence's last word
//     writes its count.
//
// Grid barriers use a 64-bit arrival counter in the workspace with a bounded wait. The
// counter only grows (by 2 x grid per launch), so no CTA has to reset it on the way out.
#include "lsa_common.cuh"

#include <atomic>

namespace lsa {
namespace idx {

constexpr int D_I = 128;
constexpr int MAX_L = 4;
constexpr int NTHREADS = 256;
constexpr int NWARPS = NTHREADS / 32;
constexpr int WORD_ROWS = 32;                       // candidate rows per keep word
constexpr int ROW_BYTES = D_I * 2;                  // one K_idx row, bf16
constexpr int ROW_STRIDE = ROW_BYTES + 16;          // padded row in shared memory: the
                                                    // 16-byte pieces lanes read at once
                                                    // fall in different banks
constexpr int WORD_SMEM = WORD_ROWS * ROW_STRIDE;   // 8.5 KB
constexpr int CHUNK_WORDS = 20;                     // K_idx words resident at once (170 KB)
constexpr int NPART = 4;                            // projection: parts per dot product
constexpr int RMAX = 4;                             // projection: W_q rows per round
constexpr int BCH = 32;                             // projection: sequences per round
constexpr int MAX_GRID = 1024;
constexpr int KW = 4;                               // warps that copy K_idx rows (named barrier 2)

struct Args {
  const uint16_t* h;         // [L][B][D]
  const uint16_t* w_q;       // [L][D_I][D]; with the factorised encoder W_2 [L][D_I][r]
  const uint16_t* w_1;       // nullable: factorised encoder, W_1 [L][r][D]
  float* u;                  // workspace [L][B][r]: the latent W_1 h (factorised encoder)
  int r;                     // latent width of the factorised encoder (0: none)
  const float* bias;         // [B]
  const uint16_t* k_idx;     // [rows][D_I]; table t of per-layer keys at row t * kls
  long long kls;             // rows between the per-layer key tables (0: one shared table)
  int lk;                    // key tables read per candidate: 1 (shared) or L
  const int64_t* kidx_off;   // [B]
  const int32_t* n_cand;     // [B]
  float* q;                  // workspace [L][B][D_I]
  uint32_t* words;           // workspace [B][n_words]: OR keep bits
  unsigned long long* sync;  // workspace: grid-barrier arrivals (grows by one grid size
                             // per barrier: 2 per launch, 3 with the factorised encoder)
  int32_t* sel_ids;          // [B][cap]
  int32_t* sel_cnt;          // [B]
  float* logits;             // nullable [L][B][max_cand]
  uint32_t* layer_mask;      // nullable [L+1][B][mask_words]
  int32_t* err;
  int B, L, D, max_cand, n_words, mask_words, cap;
  float inv_sqrt_di;
};

// Sequences met by a range of words (at most CHUNK_WORDS words, so at most as many
// sequences): first word index, words, candidates, K_idx row of block 0, bias.
struct SeqTab {
  int n;
  int b[CHUNK_WORDS];
  long long w0[CHUNK_WORDS];
  int nw[CHUNK_WORDS];
  int nc[CHUNK_WORDS];
  long long row0[CHUNK_WORDS];
  float bias[CHUNK_WORDS];
  int resume_b;              // walk state for the next range
  long long resume_base;
};

struct Smem {
  uint8_t kbuf[CHUNK_WORDS * WORD_SMEM];
  int abort;
  uint32_t own[CHUNK_WORDS];             // keep words of the first chunk, as scored
  int word_seq[CHUNK_WORDS];             // table entry of each word of the chunk
  alignas(16) float qs[CHUNK_WORDS][MAX_L][D_I];   // queries of the chunk's sequences
  int red[NWARPS];
  SeqTab tab;
  float part[RMAX][BCH][NPART];          // projection partial sums
  long long nw_total;
};

static_assert(sizeof(Smem) + 128 <= 227 * 1024, "shared memory per CTA");
// the factorised encoder stages hidden states of up to 16,384 elements in the query buffer
static_assert(sizeof(float) * CHUNK_WORDS * MAX_L * D_I >= 16384 * 2, "hidden-state staging");

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Candidates of sequence b, clamped to [0, max_cand] (out-of-range counts are reported
// by the CTA that `report`s).
__device__ __forceinline__ int seq_cand(const Args& a, int b, bool report) {
  int n = __ldg(a.n_cand + b);
  if (n < 0 || n > a.max_cand) {
    if (report) set_err(a.err, LSA_DEVERR_BAD_SIZE);
    n = n < 0 ? 0 : a.max_cand;
  }
  return n;
}
__device__ __forceinline__ int seq_words(int n) { return (n + WORD_ROWS - 1) / WORD_ROWS; }

// Candidate count, K_idx offset and bias of sequence `lane` (< 32), loaded together.
struct SeqHead {
  int n;
  long long row0;
  float bias;
};

// Total keep words of the batch, summed by one warp (every lane gets it). The first 32
// sequences' counts, K_idx offsets and biases, which the plan reads next, are loaded in
// the same round trip and returned in `head`.
__device__ __forceinline__ long long warp_total_words(const Args& a, int lane, SeqHead& head) {
  head.n = 0;
  head.row0 = 0;
  head.bias = 0.f;
  if (lane < a.B) {
    head.n = seq_cand(a, lane, false);
    head.row0 = __ldg(a.kidx_off + lane);
    head.bias = __ldg(a.bias + lane);
  }
  long long s = seq_words(head.n);
  for (int b = lane + 32; b < a.B; b += 32) s += seq_words(seq_cand(a, b, false));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

// Warp 0: fill t with the sequences that own words of [w_lo, w_hi), walking forward
// from the saved state (sequence resume_b, whose first word is resume_base). `head`, if
// given, holds sequence `lane`'s count, offset and bias (the walk's first 32 sequences).
__device__ __forceinline__ void plan_words(const Args& a, long long w_lo, long long w_hi, SeqTab* t,
                                          int lane, const SeqHead* head = nullptr) {
  int found = 0;
  long long base = t->resume_base;
  int last_b = t->resume_b;
  long long last_base = t->resume_base;
  for (int b0 = t->resume_b; b0 < a.B && base < w_hi; b0 += 32) {
    const int b = b0 + lane;
    const bool pre = head != nullptr && b0 == 0;
    const int n = pre ? head->n : (b < a.B ? seq_cand(a, b, false) : 0);
    const long long row0 = pre ? head->row0 : (b < a.B ? __ldg(a.kidx_off + b) : 0);
    const float bias = pre ? head->bias : (b < a.B ? __ldg(a.bias + b) : 0.f);
    const int nw = seq_words(n);
    long long incl = nw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const long long p = base + incl - nw;     // first word of sequence b
    const bool hit = nw > 0 && p < w_hi && p + nw > w_lo;
    const unsigned mask = __ballot_sync(0xffffffffu, hit);
    if (hit) {
      const int i = found + __popc(mask & ((1u << lane) - 1u));
      if (i < CHUNK_WORDS) {
        t->b[i] = b;
        t->w0[i] = p;
        t->nw[i] = nw;
        t->nc[i] = n;
        t->row0[i] = row0;
        t->bias[i] = bias;
      }
    }
    if (mask != 0) {
      const int hi_lane = 31 - __clz(mask);
      last_b = __shfl_sync(0xffffffffu, b, hi_lane);
      last_base = __shfl_sync(0xffffffffu, p, hi_lane);
    }
    found += __popc(mask);
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    t->n = found < CHUNK_WORDS ? found : CHUNK_WORDS;
    t->resume_b = last_b;          // the last sequence met may continue into the next range
    t->resume_base = last_base;
  }
}

// Bounded spin until the 64-bit *counter >= target (acquire, gpu scope), with the same
// two limits as the 32-bit spin_until_geq: the timer and an iteration count that the
// sleep between polls makes longer than limit_ns.
__device__ __forceinline__ bool spin_until_geq64(const unsigned long long* counter,
                                                 unsigned long long target,
                                                 uint64_t limit_ns = LSA_WAIT_LIMIT_NS) {
  const uint64_t t0 = globaltimer_ns();
  const uint64_t max_polls = limit_ns / 16u + 1024u;
  for (uint64_t it = 0;; ++it) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(counter) : "memory");
    if (v >= target) return true;
    if (it >= 64) __nanosleep(32);   // the first polls back to back: barriers are short
    if (globaltimer_ns() - t0 > limit_ns || it > max_polls) return false;
  }
}

// Grid-wide barrier on a 64-bit arrival counter that only grows: every launch adds
// exactly 2 x gridDim.x (each CTA arrives at both barriers, also after giving up), so at
// a barrier the count it must reach is the next multiple of gridDim.x above the value
// this CTA's arrival saw. Nothing has to reset the counter after the launch. The wait is
// bounded; once the CTA has given up (abort) it still arrives but no longer waits.
__device__ __forceinline__ void grid_sync(const Args& a, Smem* s) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned long long seen = atomicAdd(a.sync, 1ull);
    const unsigned long long target = (seen / gridDim.x + 1ull) * gridDim.x;
    if (!s->abort && !spin_until_geq64(a.sync, target)) {
      set_err(a.err, LSA_DEVERR_TIMEOUT);
      s->abort = 1;
    }
    __threadfence();
  }
  __syncthreads();
}

// Warp 0: plan the chunk [cw0, cw1) of keep words into s->tab and s->word_seq.
__device__ __forceinline__ void plan_chunk(const Args& a, Smem* s, long long cw0, long long cw1,
                                           int lane, const SeqHead* head = nullptr) {
  plan_words(a, cw0, cw1, &s->tab, lane, head);
  __syncwarp();
  const int nwc = static_cast<int>(cw1 - cw0);
  if (lane < nwc) {
    const long long w = cw0 + lane;
    int i = 0;
    while (i + 1 < s->tab.n && s->tab.w0[i + 1] <= w) ++i;
    s->word_seq[lane] = i;
  }
}

// Copy warps (thread ct of KW * 32): start the 16-byte asynchronous copies of the planned
// chunk's K_idx rows into s->kbuf (padded rows; a sequence's last word may be partial).
// Each copy warp completes its own copies with cp_async_wait_all.
__device__ __forceinline__ void copy_chunk(const Args& a, Smem* s, long long cw0, long long cw1,
                                           int ct) {
  const int nwc = static_cast<int>(cw1 - cw0);
  for (int k = 0; k < nwc; ++k) {
    const int i = s->word_seq[k];
    const int wi = static_cast<int>(cw0 + k - s->tab.w0[i]);
    const int rows = min(WORD_ROWS, s->tab.nc[i] - WORD_ROWS * wi);
    for (int t = 0; t < a.lk; ++t) {       // the word's rows of each key table
      const uint8_t* src = reinterpret_cast<const uint8_t*>(
          a.k_idx + (t * a.kls + s->tab.row0[i] + static_cast<long long>(WORD_ROWS) * wi) * D_I);
      const uint32_t dst = smem_u32(s->kbuf + (k * a.lk + t) * WORD_SMEM);
      for (int p = ct; p < rows * (ROW_BYTES / 16); p += KW * 32) {
        const int r = p >> 4, c = p & 15;
        cp_async16(dst + r * ROW_STRIDE + c * 16, src + r * ROW_BYTES + c * 16);
      }
    }
  }
  cp_async_commit();
}

// All threads: stage the queries of the chunk's sequences in shared memory (one round
// trip to L2 for the whole CTA).
__device__ __forceinline__ void stage_queries(const Args& a, Smem* s) {
  const int per_seq = a.L * (D_I / 4);                  // float4s per sequence
  const int total = s->tab.n * per_seq;
  for (int i = threadIdx.x; i < total; i += NTHREADS) {
    const int e = i / per_seq, r = i - e * per_seq;
    const int l = r / (D_I / 4), c4 = r - l * (D_I / 4);
    const float4 v = __ldcg(reinterpret_cast<const float4*>(
                                a.q + (static_cast<long long>(l) * a.B + s->tab.b[e]) * D_I) + c4);
    *reinterpret_cast<float4*>(&s->qs[e][l][4 * c4]) = v;
  }
}

// Warp: keep word k of the current chunk, one lane per candidate row. The row's 16
// pieces of 8 elements are read from its padded shared-memory row, the queries' pieces
// are shared-memory broadcasts; each layer's dot product runs in two interleaved chains
// joined in a fixed order. One ballot per layer gives the word's keep bits; the OR over
// the NL (= L) layers is returned. NL is a template argument so that the layers' chains
// form one straight-line block the scheduler can interleave.
template <bool PER_LAYER, int NL>
__device__ __forceinline__ uint32_t score_word(const Args& a, Smem* s, int k, long long cw0, int lane) {
  const int i = s->word_seq[k];
  const int wi = static_cast<int>(cw0 + k - s->tab.w0[i]);
  const int c = WORD_ROWS * wi + lane;
  const bool valid = c < s->tab.nc[i];
  const float bias = s->tab.bias[i];
  const int b = s->tab.b[i];
  const uint8_t* rp = s->kbuf + k * a.lk * WORD_SMEM + lane * ROW_STRIDE;
  float acc[NL][2];
#pragma unroll
  for (int l = 0; l < NL; ++l) acc[l][0] = acc[l][1] = 0.f;
#pragma unroll 4
  for (int j = 0; j < D_I / 8; ++j) {
    float kf[8];
    if (!PER_LAYER) unpack8(*reinterpret_cast<const uint4*>(rp + 16 * j), kf);
#pragma unroll
    for (int l = 0; l < NL; ++l) {
      if (PER_LAYER) unpack8(*reinterpret_cast<const uint4*>(rp + l * WORD_SMEM + 16 * j), kf);
      const float4 qa = *reinterpret_cast<const float4*>(&s->qs[i][l][8 * j]);
      const float4 qb = *reinterpret_cast<const float4*>(&s->qs[i][l][8 * j + 4]);
      float& u = acc[l][j & 1];
      u = fmaf(qa.x, kf[0], u);
      u = fmaf(qa.y, kf[1], u);
      u = fmaf(qa.z, kf[2], u);
      u = fmaf(qa.w, kf[3], u);
      u = fmaf(qb.x, kf[4], u);
      u = fmaf(qb.y, kf[5], u);
      u = fmaf(qb.z, kf[6], u);
      u = fmaf(qb.w, kf[7], u);
    }
  }
  uint32_t wor = 0;
  uint32_t wl[NL];
#pragma unroll
  for (int l = 0; l < NL; ++l) {
    const float z = fmaf(acc[l][0] + acc[l][1], a.inv_sqrt_di, bias);
    if (a.logits != nullptr && valid)
      a.logits[(static_cast<long long>(l) * a.B + b) * a.max_cand + c] = z;
    wl[l] = __ballot_sync(0xffffffffu, valid && z > 0.f);
    wor |= wl[l];
  }
  if (lane == 0) {
    a.words[static_cast<long long>(b) * a.n_words + wi] = wor;
    if (a.layer_mask != nullptr) {
#pragma unroll
      for (int l = 0; l < NL; ++l)
        a.layer_mask[(static_cast<long long>(l) * a.B + b) * a.mask_words + wi] = wl[l];
      a.layer_mask[(static_cast<long long>(NL) * a.B + b) * a.mask_words + wi] = wor;
    }
  }
  return wor;
}

template <bool PER_LAYER>
__device__ __forceinline__ uint32_t score_word_any(const Args& a, Smem* s, int k, long long cw0,
                                                   int lane) {
  switch (a.L) {
    case 1: return score_word<PER_LAYER, 1>(a, s, k, cw0, lane);
    case 2: return score_word<PER_LAYER, 2>(a, s, k, cw0, lane);
    case 3: return score_word<PER_LAYER, 3>(a, s, k, cw0, lane);
    default: return score_word<PER_LAYER, MAX_L>(a, s, k, cw0, lane);
  }
}

// Warps KW.. (PROJ_THREADS threads, named barrier 1): q rows [r_lo, r_hi) of the stacked
// W_q (row = l * D_I + j) for every sequence. Each dot product is cut into NPART parts of
// whole 8-element groups; a warp sums one part (lane-strided, then a butterfly), and the
// parts are added in order. The input vector is h (bf16, D wide) or, for the factorised
// encoder's second stage, the fp32 latent u (r wide, written earlier in this launch, so
// it is read through L2).
constexpr int PROJ_THREADS = NTHREADS - 32 * KW;
constexpr int PROJ_WARPS = PROJ_THREADS / 32;

template <bool F32_IN>
__device__ __forceinline__ void load8(const Args& a, int l, int b, int n, int g, float (&f)[8]) {
  if constexpr (F32_IN) {
    const float4* v = reinterpret_cast<const float4*>(a.u + (static_cast<long long>(l) * a.B + b) * n) + 2 * g;
    const float4 x = __ldcg(v), y = __ldcg(v + 1);
    f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
    f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
  } else {
    const uint4* v = reinterpret_cast<const uint4*>(a.h + (static_cast<long long>(l) * a.B + b) * n);
    unpack8(__ldg(v + g), f);
  }
}

template <bool F32_IN>
__device__ __forceinline__ void project_rows(const Args& a, Smem* s, int r_lo, int r_hi) {
  const int tid = threadIdx.x - 32 * KW, warp = tid >> 5, lane = tid & 31;
  const int n = F32_IN ? a.r : a.D;
  const int g8 = n / 8;
  for (int rg = r_lo; rg < r_hi; rg += RMAX) {
    const int nr = min(RMAX, r_hi - rg);
    for (int b0 = 0; b0 < a.B; b0 += BCH) {
      const int nb = min(BCH, a.B - b0);
      const int tasks = nr * nb * NPART;
      for (int t = warp; t < tasks; t += PROJ_WARPS) {
        const int p = t % NPART;
        const int rb = t / NPART;
        const int bl = rb % nb, r = rb / nb;
        const int row = rg + r;
        const int l = row / D_I;
        const uint4* wrow = reinterpret_cast<const uint4*>(a.w_q + static_cast<long long>(row) * n);
        const int g_lo = (p * g8) / NPART, g_hi = ((p + 1) * g8) / NPART;
        float acc = 0.f;
#pragma unroll 4
        for (int g = g_lo + lane; g < g_hi; g += 32) {
          float wf[8], hf[8];
          unpack8(__ldg(wrow + g), wf);
          load8<F32_IN>(a, l, b0 + bl, n, g, hf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc = fmaf(wf[e], hf[e], acc);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) s->part[r][bl][p] = acc;
      }
      named_bar_sync(1, PROJ_THREADS);
      for (int i = tid; i < nr * nb; i += PROJ_THREADS) {
        const int r = i / nb, bl = i % nb;
        float sum = 0.f;
#pragma unroll
        for (int p = 0; p < NPART; ++p) sum += s->part[r][bl][p];
        const int row = rg + r;
        const int l = row / D_I, j = row % D_I;
        a.q[(static_cast<long long>(l) * a.B + b0 + bl) * D_I + j] = sum;
      }
      named_bar_sync(1, PROJ_THREADS);
    }
  }
}

// First stage of the factorised encoder, all NTHREADS threads: u[l][b][k] = W_1[l][k] .
// h[l][b] in fp32 for the rows [k_lo, k_hi) of the stacked W_1 (row = l * r + k), one warp
// per row at a time. The hidden states of a layer are staged in shared memory a group of
// up to LR_SEQ sequences at a time (the query buffer is idle in this phase); each lane
// keeps its slice of the W_1 row in registers while it serves the whole group, and a
// row's dot product is the lanes' fixed-order partial sums joined by a butterfly.
constexpr int LR_BATCH = 16;                        // 16-byte W_1 pieces per lane in flight
constexpr int LR_SEQ = 4;                           // sequences per staged group
__device__ __forceinline__ void lowrank_rows(const Args& a, Smem* s, int k_lo, int k_hi) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4* hs = reinterpret_cast<uint4*>(&s->qs[0][0][0]);
  constexpr int HS_CAP = static_cast<int>(sizeof(s->qs) / sizeof(uint4));   // 16-byte slots
  const int g8 = a.D / 8;                           // 16-byte pieces per row (<= HS_CAP)
  const int gsz = max(1, min(LR_SEQ, HS_CAP / g8)); // sequences staged at once
  int row = k_lo;
  while (row < k_hi) {
    const int l = row / a.r;
    const int seg_hi = min(k_hi, (l + 1) * a.r);   // this range's rows of layer l
    for (int b0 = 0; b0 < a.B; b0 += gsz) {
      const int nb = min(gsz, a.B - b0);
      __syncthreads();                              // the previous group's readers are done
      const uint4* src = reinterpret_cast<const uint4*>(a.h + (static_cast<long long>(l) * a.B + b0) * a.D);
      for (int i = threadIdx.x; i < nb * g8; i += NTHREADS) hs[i] = __ldg(src + i);
      __syncthreads();
      // two rows per warp at a time, all their 16-byte pieces requested before any use
      for (int k = row + 2 * warp; k < seg_hi; k += 2 * NWARPS) {
        const bool two = k + 1 < seg_hi;
        const uint4* wrow0 = reinterpret_cast<const uint4*>(a.w_1 + static_cast<long long>(k) * a.D);
        const uint4* wrow1 = reinterpret_cast<const uint4*>(a.w_1 + static_cast<long long>(two ? k + 1 : k) * a.D);
        float acc0[LR_SEQ], acc1[LR_SEQ];
#pragma unroll
        for (int e = 0; e < LR_SEQ; ++e) acc0[e] = acc1[e] = 0.f;
        for (int g0 = 0; g0 < g8; g0 += 32 * LR_BATCH) {
          uint4 w0[LR_BATCH], w1[LR_BATCH];
#pragma unroll
          for (int t = 0; t < LR_BATCH; ++t) {
            const int g = g0 + lane + 32 * t;
            w0[t] = g < g8 ? __ldg(wrow0 + g) : make_uint4(0u, 0u, 0u, 0u);
            w1[t] = (g < g8 && two) ? __ldg(wrow1 + g) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int t = 0; t < LR_BATCH; ++t) {
            const int g = g0 + lane + 32 * t;
            if (g < g8) {
              float wf0[8], wf1[8];
              unpack8(w0[t], wf0);
              unpack8(w1[t], wf1);
#pragma unroll
              for (int e = 0; e < LR_SEQ; ++e) {
                if (e < nb) {
                  float hf[8];
                  unpack8(hs[e * g8 + g], hf);
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    acc0[e] = fmaf(wf0[i], hf[i], acc0[e]);
                    acc1[e] = fmaf(wf1[i], hf[i], acc1[e]);
                  }
                }
              }
            }
          }
        }
#pragma unroll
        for (int e = 0; e < LR_SEQ; ++e) {
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) {
            acc0[e] += __shfl_xor_sync(0xffffffffu, acc0[e], o);
            acc1[e] += __shfl_xor_sync(0xffffffffu, acc1[e], o);
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int e = 0; e < LR_SEQ; ++e) {
            if (e < nb) {
              float* ub = a.u + (static_cast<long long>(l) * a.B + b0 + e) * a.r - static_cast<long long>(l) * a.r;
              ub[k] = acc0[e];
              if (two) ub[k + 1] = acc1[e];
            }
          }
        }
      }
    }
    row = seg_hi;
  }
}

// Warp 0: ids of the keep words [dw0, dw1) (at most CHUNK_WORDS, planned in s->tab).
// `carry` = kept blocks of the chunk's first sequence in words before dw0; returns the
// same for the next chunk. The chunk's first `own_n` words are read from s->own.
__device__ __forceinline__ int compact_chunk(const Args& a, Smem* s, long long dw0, long long dw1,
                                             int carry, int own_n, int lane) {
  const int nwc = static_cast<int>(dw1 - dw0);
  int i = 0, b = 0, wi = 0, ts = 0;
  uint32_t bits = 0;
  if (lane < nwc) {
    const long long w = dw0 + lane;
    while (i + 1 < s->tab.n && s->tab.w0[i + 1] <= w) ++i;
    b = s->tab.b[i];
    wi = static_cast<int>(w - s->tab.w0[i]);
    ts = s->tab.w0[i] > dw0 ? static_cast<int>(s->tab.w0[i] - dw0) : 0;  // lane of its 1st word
    bits = lane < own_n ? s->own[lane] : __ldcg(a.words + static_cast<long long>(b) * a.n_words + wi);
  }
  const int cnt = __popc(bits);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  const int excl = incl - cnt;
  const int ex_ts = __shfl_sync(0xffffffffu, excl, ts);
  const int base = (lane < nwc && s->tab.w0[i] < dw0) ? carry : 0;
  if (lane < nwc) {
    int pos = base + excl - ex_ts;
    int32_t* out = a.sel_ids + static_cast<long long>(b) * a.cap;
    uint32_t rem = bits;
    while (rem) {
      const int bit = __ffs(rem) - 1;
      rem &= rem - 1;
      if (pos < a.cap) out[pos] = WORD_ROWS * wi + bit;
      ++pos;
    }
    if (wi == s->tab.nw[i] - 1) {        // the sequence's last word: its count
      if (pos > a.cap) set_err(a.err, LSA_DEVERR_SEL_CAPACITY);
      a.sel_cnt[b] = pos < a.cap ? pos : a.cap;
    }
  }
  // the next chunk's carry: the last sequence's kept blocks so far
  const int last = nwc - 1;
  const int ts_last = __shfl_sync(0xffffffffu, ts, last);
  const int base_last = __shfl_sync(0xffffffffu, base, last);
  const int incl_last = __shfl_sync(0xffffffffu, incl, last);
  const int ex_last = __shfl_sync(0xffffffffu, excl, ts_last);
  return base_last + incl_last - ex_last;
}

__global__ void __launch_bounds__(NTHREADS, 1) index_kernel(const Args a) {
  extern __shared__ uint8_t smem_raw[];
  Smem* s = reinterpret_cast<Smem*>(smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long G = gridDim.x;
  const int cta = blockIdx.x;

  if (tid == 0) {
    s->abort = 0;
    s->tab.resume_b = 0;
    s->tab.resume_base = 0;
  }
  // Launched as a programmatic dependent: the set-up above overlaps the tail of the
  // preceding kernel; nothing it may write is read before this point.
  grid_dependency_wait();
  grid_dependents_launch();
  __syncthreads();
  // ---- phase A. Warp 0 plans this CTA's keep words [W0, W1), and the KW copy warps
  // start the first chunk's K_idx copies at once; warps KW..: this CTA's rows of q.
  const long long ccap = CHUNK_WORDS / a.lk;   // words whose key rows fit in kbuf
  if (warp < KW) {
    if (warp == 0) {
      SeqHead head;
      const long long NW = warp_total_words(a, lane, head);
      const long long W0 = (cta * NW) / G, W1 = ((cta + 1) * NW) / G;
      if (W1 > W0) plan_chunk(a, s, W0, W1 < W0 + ccap ? W1 : W0 + ccap, lane, &head);
      if (lane == 0) s->nw_total = NW;
    }
    named_bar_sync(2, KW * 32);
    const long long NW = s->nw_total;
    const long long W0 = (cta * NW) / G, W1 = ((cta + 1) * NW) / G;
    if (W1 > W0) copy_chunk(a, s, W0, W1 < W0 + ccap ? W1 : W0 + ccap, tid);
  } else if (a.w_1 == nullptr) {
    const int RQ = a.L * D_I;
    project_rows<false>(a, s, static_cast<int>((cta * RQ) / G), static_cast<int>(((cta + 1) * RQ) / G));
  }
  if (a.w_1 != nullptr) {
    // factorised encoder: the latent u = W_1 h by all warps (the copy warps join once
    // their K_idx copies are issued), a grid barrier, then q = W_2 u
    const long long RU = static_cast<long long>(a.L) * a.r;
    lowrank_rows(a, s, static_cast<int>((cta * RU) / G), static_cast<int>(((cta + 1) * RU) / G));
    grid_sync(a, s);
    if (warp >= KW && !s->abort) {
      const int RQ = a.L * D_I;
      project_rows<true>(a, s, static_cast<int>((cta * RQ) / G), static_cast<int>(((cta + 1) * RQ) / G));
    }
  }
  grid_sync(a, s);
  const long long NW = s->nw_total;
  const long long W0 = (cta * NW) / G, W1 = ((cta + 1) * NW) / G;

  // ---- phase B: keep words, one warp per word
  int chunk = 0;
  for (long long cw0 = W0; cw0 < W1; cw0 += ccap, ++chunk) {
    const long long cw1 = W1 < cw0 + ccap ? W1 : cw0 + ccap;
    if (cw0 != W0) {
      __syncthreads();                          // every warp is done with kbuf
      if (warp == 0) plan_chunk(a, s, cw0, cw1, lane);
      __syncthreads();                          // the chunk's plan is visible
      if (warp < KW) copy_chunk(a, s, cw0, cw1, tid);
    }
    if (warp < KW) cp_async_wait_all();         // the chunk's rows (each copy warp's own)
    if (!s->abort) stage_queries(a, s);
    __syncthreads();
    if (s->abort) break;
    const int nwc = static_cast<int>(cw1 - cw0);
    for (int k = warp; k < nwc; k += NWARPS) {
      const uint32_t wor = a.lk > 1 ? score_word_any<true>(a, s, k, cw0, lane)
                                    : score_word_any<false>(a, s, k, cw0, lane);
      if (lane == 0 && chunk == 0) s->own[k] = wor;
    }
  }
  grid_sync(a, s);

  // ---- phase C: ordered ids
  if (!s->abort && W1 > W0) {            // the same branch in every thread of the CTA
    // The plan of [W0, W1) made in phase A is still in s->tab when phase B had one chunk.
    if (warp == 0 && W1 - W0 > ccap) {
      s->tab.resume_b = 0;
      s->tab.resume_base = 0;
      plan_words(a, W0, W1 < W0 + CHUNK_WORDS ? W1 : W0 + CHUNK_WORDS, &s->tab, lane);
    }
    __syncthreads();
    // kept blocks of the first sequence in its words before W0, summed by the CTA
    int part = 0;
    const long long first = s->tab.w0[0];
    if (first < W0) {
      const long long wrow = static_cast<long long>(s->tab.b[0]) * a.n_words;
      const int skip = static_cast<int>(W0 - first);
      for (int w = tid; w < skip; w += NTHREADS) part += __popc(__ldcg(a.words + wrow + w));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) s->red[warp] = part;
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
#pragma unroll
      for (int w = 0; w < NWARPS; ++w) carry += s->red[w];
      for (long long dw0 = W0; dw0 < W1; dw0 += CHUNK_WORDS) {
        const long long dw1 = W1 < dw0 + CHUNK_WORDS ? W1 : dw0 + CHUNK_WORDS;
        if (dw0 != W0) {
          plan_words(a, dw0, dw1, &s->tab, lane);
          __syncwarp();
        }
        const int own_n = dw0 == W0 ? static_cast<int>(W1 - W0 < ccap ? W1 - W0 : ccap) : 0;
        carry = compact_chunk(a, s, dw0, dw1, carry, own_n, lane);
        __syncwarp();
      }
    }
  }

  // sequences without candidates get a zero count; bad counts are reported once
  for (long long b = static_cast<long long>(cta) * NTHREADS + tid; b < a.B; b += G * NTHREADS) {
    if (seq_cand(a, static_cast<int>(b), true) == 0) a.sel_cnt[b] = 0;
  }
}

}  // namespace idx
}  // namespace lsa

// ------------------------------------------------------------------------ host side
namespace {
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace: the 64-bit grid-barrier counter on its own 256-byte line at the start (zero
// before the first call; each call adds one grid size per barrier), then q fp32
// [L][B][d_i], the keep words u32 [B][n_words] and, for the factorised encoder, the latent
// u fp32 [L][B][r]. The counter's place does not depend on the shape.
struct IndexWsLayout {
  size_t q_off, words_off, u_off, sync_off, total;
  int n_words;
};

IndexWsLayout index_ws_layout(int B, int L, int max_cand, int r) {
  IndexWsLayout s;
  s.n_words = (max_cand + 31) / 32;
  if (s.n_words < 1) s.n_words = 1;
  s.sync_off = 0;
  s.q_off = 256;
  s.words_off = align256(s.q_off + static_cast<size_t>(L) * B * lsa::idx::D_I * sizeof(float));
  s.u_off = align256(s.words_off + static_cast<size_t>(B) * s.n_words * sizeof(uint32_t));
  s.total = align256(s.u_off + static_cast<size_t>(L) * B * (r > 0 ? r : 0) * sizeof(float));
  return s;
}

constexpr size_t kIndexSmem = sizeof(lsa::idx::Smem) + 128;   // + alignment slack
}  // namespace

extern "C" size_t lsa_index_workspace_size(int32_t B, int32_t L, int32_t d_i, int32_t max_cand) {
  if (B <= 0 || L <= 0 || d_i != lsa::idx::D_I || max_cand < 0) return 0;
  return index_ws_layout(B, L, max_cand, 0).total;
}

namespace {
// One indexer launch. w_1 == nullptr: the query encoders are w_q [L][d_i][D]; otherwise
// they are factorised, w_1 [L][r][D] then w_q = W_2 [L][d_i][r].
lsa_status index_launch(const uint16_t* h, const uint16_t* w_q, const uint16_t* w_1, int32_t r,
                        const float* bias, const uint16_t* k_idx, int64_t kidx_layer_stride,
                        const int64_t* kidx_off, const int32_t* n_cand, int32_t B, int32_t L,
                        int32_t D, int32_t d_i, int32_t max_cand, int32_t* sel_ids,
                        int32_t* sel_cnt, int32_t cap, float* logits, uint32_t* layer_mask,
                        void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  if (!h || !w_q || !bias || !k_idx || !kidx_off || !n_cand || !sel_cnt || !ws || !err)
    return LSA_ERR_INVALID_ARG;
  if (kidx_layer_stride < 0) return LSA_ERR_INVALID_ARG;
  if (cap > 0 && !sel_ids) return LSA_ERR_INVALID_ARG;
  if (B <= 0 || B > 65535 || L < 1 || L > lsa::idx::MAX_L || d_i != lsa::idx::D_I || D <= 0 ||
      D % 256 != 0 || max_cand < 0 || cap < 0)
    return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w_q) |
       reinterpret_cast<uintptr_t>(k_idx) | reinterpret_cast<uintptr_t>(ws)) & 15u)
    return LSA_ERR_INVALID_ARG;
  if (w_1 != nullptr && (r < 256 || r > 8192 || r % 256 != 0 || D > 16384 ||
                        (reinterpret_cast<uintptr_t>(w_1) & 15u)))
    return LSA_ERR_INVALID_ARG;
  const IndexWsLayout lay = index_ws_layout(B, L, max_cand, w_1 != nullptr ? r : 0);
  if (ws_bytes < lay.total) return LSA_ERR_INVALID_ARG;
  const int n_sm = lsa_host::sm_count();
  if (n_sm <= 0) return LSA_ERR_CUDA;
  const int G = n_sm < lsa::idx::MAX_GRID ? n_sm : lsa::idx::MAX_GRID;

  {
    const lsa_status st = lsa_host::ensure_smem_limit(
        reinterpret_cast<const void*>(lsa::idx::index_kernel), static_cast<int>(kIndexSmem));
    if (st != LSA_OK) return st;
  }
  uint8_t* base = static_cast<uint8_t*>(ws);
  lsa::idx::Args a;
  a.h = h;
  a.w_q = w_q;
  a.w_1 = w_1;
  a.r = w_1 != nullptr ? r : 0;
  a.u = w_1 != nullptr ? reinterpret_cast<float*>(base + lay.u_off) : nullptr;
  a.bias = bias;
  a.k_idx = k_idx;
  a.kls = kidx_layer_stride;
  a.lk = kidx_layer_stride > 0 ? L : 1;
  a.kidx_off = kidx_off;
  a.n_cand = n_cand;
  a.q = reinterpret_cast<float*>(base + lay.q_off);
  a.words = reinterpret_cast<uint32_t*>(base + lay.words_off);
  a.sync = reinterpret_cast<unsigned long long*>(base + lay.sync_off);
  a.sel_ids = sel_ids;
  a.sel_cnt = sel_cnt;
  a.logits = logits;
  a.layer_mask = layer_mask;
  a.err = err;
  a.B = B;
  a.L = L;
  a.D = D;
  a.max_cand = max_cand;
  a.n_words = lay.n_words;
  a.mask_words = (max_cand + 31) / 32;
  a.cap = cap;
  a.inv_sqrt_di = 1.0f / sqrtf(static_cast<float>(d_i));

  // Cooperative launch: the G CTAs (one per SM) are resident together, which the two
  // grid barriers rely on.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(lsa::idx::NTHREADS);
  cfg.dynamicSmemBytes = kIndexSmem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  // A programmatic dependent as well, so that the CTAs' set-up overlaps the preceding
  // kernel's tail; a device that refuses the combination gets plain cooperative launches.
  static std::atomic<int> pdl_state[64];   // 0 unknown/accepted, 1 refused (per device)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  const bool pdl = pdl_state[dev].load(std::memory_order_relaxed) == 0;
  cfg.numAttrs = pdl ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, lsa::idx::index_kernel, a);
  if (e == cudaErrorNotSupported && pdl) {
    cudaGetLastError();
    pdl_state[dev].store(1, std::memory_order_relaxed);
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, lsa::idx::index_kernel, a);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

}  // namespace

extern "C" lsa_status lsa_index_ex(const uint16_t* h, const uint16_t* w_q, const float* bias,
                                   const uint16_t* k_idx, int64_t kidx_layer_stride,
                                   const int64_t* kidx_off, const int32_t* n_cand, int32_t B,
                                   int32_t L, int32_t D, int32_t d_i, int32_t max_cand,
                                   int32_t* sel_ids, int32_t* sel_cnt, int32_t cap, float* logits,
                                   uint32_t* layer_mask, void* ws, size_t ws_bytes, int32_t* err,
                                   void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_index");
  return index_launch(h, w_q, nullptr, 0, bias, k_idx, kidx_layer_stride, kidx_off, n_cand, B, L,
                      D, d_i, max_cand, sel_ids, sel_cnt, cap, logits, layer_mask, ws, ws_bytes,
                      err, stream);
}

extern "C" size_t lsa_index_lowrank_workspace_size(int32_t B, int32_t L, int32_t d_i, int32_t r,
                                                   int32_t max_cand) {
  if (B <= 0 || L <= 0 || d_i != lsa::idx::D_I || r <= 0 || max_cand < 0) return 0;
  return index_ws_layout(B, L, max_cand, r).total;
}

extern "C" lsa_status lsa_index_lowrank(const uint16_t* h, const uint16_t* w_1,
                                        const uint16_t* w_2, int32_t r, const float* bias,
                                        const uint16_t* k_idx, int64_t kidx_layer_stride,
                                        const int64_t* kidx_off, const int32_t* n_cand,
                                        int32_t B, int32_t L, int32_t D, int32_t d_i,
                                        int32_t max_cand, int32_t* sel_ids, int32_t* sel_cnt,
                                        int32_t cap, float* logits, uint32_t* layer_mask,
                                        void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  lsa_host::NvtxRange nvtx_range("lsa_index_lowrank");
  if (!w_1 || !w_2) return LSA_ERR_INVALID_ARG;
  return index_launch(h, w_2, w_1, r, bias, k_idx, kidx_layer_stride, kidx_off, n_cand, B, L, D,
                      d_i, max_cand, sel_ids, sel_cnt, cap, logits, layer_mask, ws, ws_bytes, err,
                      stream);
}

extern "C" lsa_status lsa_index(const uint16_t* h, const uint16_t* w_q, const float* bias,
                                const uint16_t* k_idx, const int64_t* kidx_off,
                                const int32_t* n_cand, int32_t B, int32_t L, int32_t D,
                                int32_t d_i, int32_t max_cand, int32_t* sel_ids, int32_t* sel_cnt,
                                int32_t cap, float* logits, uint32_t* layer_mask, void* ws,
                                size_t ws_bytes, int32_t* err, void* stream) {
  return lsa_index_ex(h, w_q, bias, k_idx, 0, kidx_off, n_cand, B, L, D, d_i, max_cand, sel_ids,
                      sel_cnt, cap, logits, layer_mask, ws, ws_bytes, err, stream);
}
