// Neural Memory Indexer pass: query projection, block scoring, sign test, OR over the
// indexer layers, and ordered compaction of the kept block ids.
//
// "FlashMemory-DeepSeek-V4 Explained" (zhichai.net): section 2 steps 2-3 (score the
// historical blocks from the current hidden state, keep sigmoid > 0.5), section 3 (one
// small query projection per layer against frozen compressed block keys), section 4
// (independent indexers at three layers, OR-ed).
//
// Two kernels:
//  1. project: q[l][b][:] = W_q[l] . h[l][b] in fp32 (one warp per output row, bf16
//     operands read with 16-byte loads, fixed-order warp reduction);
//  2. score: 16 lanes per candidate row (16 bytes each, so a warp reads two 256-byte
//     K_idx rows per load, coalesced), z_l = q_l . k / sqrt(d_i) + bias, keep bit
//     z_l > 0 (equal to sigmoid(z_l) > 0.5), OR over the layers, packed with warp
//     ballots into 32-bit words. The last CTA of each sequence (atomic ticket, no
//     waiting) turns the words into the ascending id list with a block prefix sum.
#include "lsa_common.cuh"

namespace lsa {
namespace idx {

constexpr int D_I = 128;
constexpr int MAX_L = 4;
constexpr int PROJ_WARPS = 4;        // output rows per projection CTA
constexpr int PROJ_BCHUNK = 8;       // sequences accumulated at once per warp
constexpr int SCORE_WARPS = 8;
constexpr int ROWS_PER_CTA = SCORE_WARPS * 32;

struct Ws {
  float* q;            // [L][B][D_I]
  uint32_t* words;     // [B][n_words]   OR keep bits
  int32_t* ticket;     // [B]
};

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// q[l][b][j] = sum_i W_q[l][j][i] * h[l][b][i]
__global__ void __launch_bounds__(PROJ_WARPS * 32)
    project_kernel(const uint16_t* __restrict__ h, const uint16_t* __restrict__ w_q, int B, int L,
                   int D, float* __restrict__ q) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * PROJ_WARPS + warp;  // l * D_I + j
  if (row >= L * D_I) return;
  const int l = row / D_I, j = row % D_I;
  const uint4* wrow = reinterpret_cast<const uint4*>(w_q + static_cast<size_t>(row) * D);
  const int n_it = D / 256;
  for (int b0 = 0; b0 < B; b0 += PROJ_BCHUNK) {
    float acc[PROJ_BCHUNK];
#pragma unroll
    for (int k = 0; k < PROJ_BCHUNK; ++k) acc[k] = 0.f;
#pragma unroll 4
    for (int it = 0; it < n_it; ++it) {
      float wf[8];
      unpack8(__ldg(wrow + it * 32 + lane), wf);
#pragma unroll
      for (int k = 0; k < PROJ_BCHUNK; ++k) {
        const int b = b0 + k;
        if (b < B) {
          const uint4* hrow =
              reinterpret_cast<const uint4*>(h + (static_cast<size_t>(l) * B + b) * D);
          float hf[8];
          unpack8(__ldg(hrow + it * 32 + lane), hf);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[k] = fmaf(wf[e], hf[e], acc[k]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < PROJ_BCHUNK; ++k) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int k = 0; k < PROJ_BCHUNK; ++k)
        if (b0 + k < B) q[(static_cast<size_t>(l) * B + b0 + k) * D_I + j] = acc[k];
    }
  }
}

struct ScoreArgs {
  const uint16_t* k_idx;
  const int64_t* kidx_off;
  const int32_t* n_cand;
  const float* bias;
  const float* q;          // [L][B][D_I]
  uint32_t* words;         // [B][n_words]
  int32_t* ticket;         // [B]
  int32_t* sel_ids;        // [B][cap]
  int32_t* sel_cnt;        // [B]
  float* logits;           // nullable [L][B][max_cand]
  uint32_t* layer_mask;    // nullable [L+1][B][n_words]
  int32_t* err;
  int B, L, max_cand, n_words, mask_words, cap;
  float inv_sqrt_di;
};

__device__ __forceinline__ int clamp_cand(const ScoreArgs& a, int b, bool report) {
  int n = __ldg(a.n_cand + b);
  if (n < 0 || n > a.max_cand) {
    if (report) set_err(a.err, LSA_DEVERR_BAD_SIZE);
    n = n < 0 ? 0 : a.max_cand;
  }
  return n;
}

// grid (ceil(max_cand / ROWS_PER_CTA), B); CTA x of sequence b scores candidates
// [x*256, x*256+256) in 8 warps of 32 rows, 2 rows per load (16 lanes per row).
__global__ void __launch_bounds__(SCORE_WARPS * 32) score_kernel(const ScoreArgs a) {
  const int b = blockIdx.y;
  const int n = clamp_cand(a, b, blockIdx.x == 0 && threadIdx.x == 0);
  const int n_cta = max(1, (n + ROWS_PER_CTA - 1) / ROWS_PER_CTA);
  if (static_cast<int>(blockIdx.x) >= n_cta) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = lane >> 4, sub = lane & 15;
  const int L = a.L;
  // this lane's 8-element slice of each layer's query
  float qv[MAX_L][8];
#pragma unroll
  for (int l = 0; l < MAX_L; ++l) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      qv[l][e] = l < L ? a.q[(static_cast<size_t>(l) * a.B + b) * D_I + sub * 8 + e] : 0.f;
  }
  const float bias = __ldg(a.bias + b);
  const int c_base = blockIdx.x * ROWS_PER_CTA + warp * 32;
  const uint4* kb = reinterpret_cast<const uint4*>(a.k_idx + __ldg(a.kidx_off + b) * D_I);

  // issue all 16 loads of the warp's 32 rows first (16 B per lane each)
  uint4 kv[16];
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int c = c_base + 2 * it + half;
    kv[it] = c < n ? __ldg(kb + static_cast<size_t>(c) * (D_I / 8) + sub) : make_uint4(0, 0, 0, 0);
  }
  uint32_t w_or = 0;
  uint32_t w_l[MAX_L] = {0, 0, 0, 0};
#pragma unroll
  for (int it = 0; it < 16; ++it) {
    const int c = c_base + 2 * it + half;
    float kf[8];
    unpack8(kv[it], kf);
    bool any = false;
#pragma unroll
    for (int l = 0; l < MAX_L; ++l) {
      if (l < L) {
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(qv[l][e], kf[e], s);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float z = fmaf(s, a.inv_sqrt_di, bias);
        const bool keep = (c < n) && (z > 0.f);
        any |= keep;
        if (a.logits != nullptr && sub == 0 && c < n)
          a.logits[(static_cast<size_t>(l) * a.B + b) * a.max_cand + c] = z;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep && sub == 0);
        w_l[l] |= ((bal & 1u) << (2 * it)) | (((bal >> 16) & 1u) << (2 * it + 1));
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, any && sub == 0);
    w_or |= ((bal & 1u) << (2 * it)) | (((bal >> 16) & 1u) << (2 * it + 1));
  }
  const int word = c_base >> 5;
  if (lane == 0 && c_base < n) {
    a.words[static_cast<size_t>(b) * a.n_words + word] = w_or;
    if (a.layer_mask != nullptr) {
      for (int l = 0; l < L; ++l)
        a.layer_mask[(static_cast<size_t>(l) * a.B + b) * a.mask_words + word] = w_l[l];
      a.layer_mask[(static_cast<size_t>(L) * a.B + b) * a.mask_words + word] = w_or;
    }
  }

  // ---- last CTA of this sequence compacts the id list (no CTA ever waits)
  __shared__ int s_last;
  __shared__ int s_warp[SCORE_WARPS];
  __shared__ int s_carry;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int t = atomicAdd(a.ticket + b, 1);
    s_last = (t == n_cta - 1);
    s_carry = 0;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int n_w = (n + 31) >> 5;
  const uint32_t* words = a.words + static_cast<size_t>(b) * a.n_words;
  int32_t* out = a.sel_ids + static_cast<size_t>(b) * a.cap;
  for (int w0 = 0; w0 < n_w; w0 += SCORE_WARPS * 32) {
    const int w = w0 + threadIdx.x;
    const uint32_t bits = w < n_w ? __ldcg(words + w) : 0u;
    const int cnt = __popc(bits);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int before = s_carry;
    for (int k = 0; k < warp; ++k) before += s_warp[k];
    int pos = before + incl - cnt;
    uint32_t rem = bits;
    while (rem) {
      const int bit = __ffs(rem) - 1;
      rem &= rem - 1;
      if (pos < a.cap) out[pos] = w * 32 + bit;
      ++pos;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int k = 0; k < SCORE_WARPS; ++k) tot += s_warp[k];
      s_carry += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int total = s_carry;
    if (total > a.cap) set_err(a.err, LSA_DEVERR_SEL_CAPACITY);
    a.sel_cnt[b] = min(total, a.cap);
    a.ticket[b] = 0;  // ready for the next pass
  }
}

}  // namespace idx
}  // namespace lsa

// ------------------------------------------------------------------------ host side
namespace {
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct IndexWsLayout {
  size_t q_off, words_off, ticket_off, total;
  int n_words;
};

IndexWsLayout index_ws_layout(int B, int L, int max_cand) {
  IndexWsLayout s;
  s.n_words = (max_cand + 31) / 32;
  if (s.n_words < 1) s.n_words = 1;
  // score CTAs write whole 256-row groups: round the word count up to 8-word groups
  s.n_words = (s.n_words + 7) / 8 * 8;
  s.q_off = 0;
  s.words_off = align256(s.q_off + static_cast<size_t>(L) * B * lsa::idx::D_I * sizeof(float));
  s.ticket_off = align256(s.words_off + static_cast<size_t>(B) * s.n_words * sizeof(uint32_t));
  s.total = align256(s.ticket_off + static_cast<size_t>(B) * sizeof(int32_t));
  return s;
}
}  // namespace

extern "C" size_t lsa_index_workspace_size(int32_t B, int32_t L, int32_t d_i, int32_t max_cand) {
  if (B <= 0 || L <= 0 || d_i != lsa::idx::D_I || max_cand < 0) return 0;
  return index_ws_layout(B, L, max_cand).total;
}

extern "C" lsa_status lsa_index(const uint16_t* h, const uint16_t* w_q, const float* bias,
                                const uint16_t* k_idx, const int64_t* kidx_off,
                                const int32_t* n_cand, int32_t B, int32_t L, int32_t D,
                                int32_t d_i, int32_t max_cand, int32_t* sel_ids, int32_t* sel_cnt,
                                int32_t cap, float* logits, uint32_t* layer_mask, void* ws,
                                size_t ws_bytes, int32_t* err, void* stream) {
  if (!h || !w_q || !bias || !k_idx || !kidx_off || !n_cand || !sel_cnt || !ws || !err)
    return LSA_ERR_INVALID_ARG;
  if (cap > 0 && !sel_ids) return LSA_ERR_INVALID_ARG;
  if (B <= 0 || B > 65535 || L < 1 || L > lsa::idx::MAX_L || d_i != lsa::idx::D_I || D <= 0 ||
      D % 256 != 0 || max_cand < 0 || cap < 0)
    return LSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(h) | reinterpret_cast<uintptr_t>(w_q) |
       reinterpret_cast<uintptr_t>(k_idx)) & 15u)
    return LSA_ERR_INVALID_ARG;
  const IndexWsLayout lay = index_ws_layout(B, L, max_cand);
  if (ws_bytes < lay.total) return LSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* q = reinterpret_cast<float*>(base + lay.q_off);

  const int rows = L * lsa::idx::D_I;
  lsa::idx::project_kernel<<<(rows + lsa::idx::PROJ_WARPS - 1) / lsa::idx::PROJ_WARPS,
                             lsa::idx::PROJ_WARPS * 32, 0, s>>>(h, w_q, B, L, D, q);
  if (cudaGetLastError() != cudaSuccess) return LSA_ERR_CUDA;

  lsa::idx::ScoreArgs a;
  a.k_idx = k_idx;
  a.kidx_off = kidx_off;
  a.n_cand = n_cand;
  a.bias = bias;
  a.q = q;
  a.words = reinterpret_cast<uint32_t*>(base + lay.words_off);
  a.ticket = reinterpret_cast<int32_t*>(base + lay.ticket_off);
  a.sel_ids = sel_ids;
  a.sel_cnt = sel_cnt;
  a.logits = logits;
  a.layer_mask = layer_mask;
  a.err = err;
  a.B = B;
  a.L = L;
  a.max_cand = max_cand;
  a.n_words = lay.n_words;
  a.mask_words = (max_cand + 31) / 32;
  a.cap = cap;
  a.inv_sqrt_di = 1.0f / sqrtf(static_cast<float>(d_i));
  const int gx = max(1, (max_cand + lsa::idx::ROWS_PER_CTA - 1) / lsa::idx::ROWS_PER_CTA);
  lsa::idx::score_kernel<<<dim3(gx, B), lsa::idx::SCORE_WARPS * 32, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
