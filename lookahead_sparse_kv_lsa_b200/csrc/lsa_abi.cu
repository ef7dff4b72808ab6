// Library-wide entry points of the LSA C ABI: status text, version, state validation,
// and the host helpers shared by the kernels' launchers.
#include "lsa_common.cuh"

#include <mutex>

namespace lsa_host {

int sm_count() {
  static int cached[64];
  static std::once_flag once;
  std::call_once(once, [] {
    for (int& c : cached) c = 0;
  });
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

lsa_status ensure_smem_limit(const void* func, int bytes) {
  struct Entry {
    int dev;
    const void* func;
    int bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int n_done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].dev == dev && done[i].func == func && done[i].bytes >= bytes) return LSA_OK;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  if (n_done < 256) done[n_done++] = Entry{dev, func, bytes};
  return LSA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

lsa_status encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                           uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                           CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return LSA_ERR_CUDA;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LSA_OK : LSA_ERR_CUDA;
}

}  // namespace lsa_host

extern "C" const char* lsa_status_str(lsa_status s) {
  switch (s) {
    case LSA_OK: return "ok";
    case LSA_ERR_INVALID_ARG: return "invalid argument";
    case LSA_ERR_CAPACITY: return "capacity exceeded";
    case LSA_ERR_CUDA: return "CUDA error";
    case LSA_ERR_TIMEOUT: return "device wait timed out";
    case LSA_ERR_UNIMPLEMENTED: return "unimplemented";
    default: return "unknown status";
  }
}

extern "C" int32_t lsa_version(void) { return 100; }

namespace {
__global__ void wait_selftest_kernel(const unsigned int* flag, unsigned int target,
                                     uint64_t limit_ns, int32_t* err) {
  if (threadIdx.x == 0 && !lsa::spin_until_geq(flag, target, limit_ns))
    lsa::set_err(err, LSA_DEVERR_TIMEOUT);
}
}  // namespace

extern "C" lsa_status lsa_wait_selftest(const uint32_t* flag, uint32_t target, int64_t limit_ns,
                                        int32_t* err, void* stream) {
  if (flag == nullptr || err == nullptr || limit_ns < 1 || limit_ns > 10000000000LL)
    return LSA_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      flag, target, static_cast<uint64_t>(limit_ns), err);
  return cudaPeekAtLastError() == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}

extern "C" lsa_status lsa_state_check(const lsa_state* st) {
  if (!st) return LSA_ERR_INVALID_ARG;
  if (st->B <= 0 || st->L < 1 || st->L > 4 || st->d_i != 128 || st->D <= 0 || st->D % 256 != 0)
    return LSA_ERR_INVALID_ARG;
  if (st->H < 1 || st->H > 64 || (st->d != 128 && st->d != 256 && st->d != 384 && st->d != 512))
    return LSA_ERR_INVALID_ARG;
  if (st->W < 0 || st->W % LSA_BLOCK != 0 || st->cap < 0 || st->max_cand < 0) return LSA_ERR_INVALID_ARG;
  if (!(st->scale > 0.f)) return LSA_ERR_INVALID_ARG;
  if (!st->w_q || !st->k_idx || !st->kidx_off || !st->bias || !st->host_pool || !st->host_blk_off ||
      !st->nb0 || !st->hbm_pool || !st->n_cand || !st->sel_cnt || !st->res_pages || !st->n_res ||
      !st->block_table || !st->n_entries || !st->tail_len || !st->index_ws || !st->attn_ws ||
      !st->err)
    return LSA_ERR_INVALID_ARG;
  if (st->cap > 0 && !st->sel_ids) return LSA_ERR_INVALID_ARG;
  const int64_t wb1 = st->W / LSA_BLOCK + 1;
  if (st->bt_stride < st->cap + wb1) return LSA_ERR_INVALID_ARG;
  if (st->n_pages < static_cast<int64_t>(st->B) * wb1 || st->host_blocks <= 0)
    return LSA_ERR_INVALID_ARG;
  if (st->index_ws_bytes < lsa_index_workspace_size(st->B, st->L, st->d_i, st->max_cand))
    return LSA_ERR_INVALID_ARG;
  if (st->kidx_layer_stride < 0) return LSA_ERR_INVALID_ARG;
  if (st->kept_cnt != nullptr) {               // resident-page reuse across passes
    if (st->cap > 0 && (!st->kept_ids || !st->kept_pages)) return LSA_ERR_INVALID_ARG;
    const int n_sm = lsa_host::sm_count();
    const int64_t sel_pages = st->n_pages - static_cast<int64_t>(st->B) * wb1;
    if (!st->gather_ws || n_sm <= 0 || sel_pages > INT32_MAX ||
        st->gather_ws_bytes < lsa_gather_delta_workspace_size(st->B, st->cap,
                                                              static_cast<int32_t>(sel_pages), n_sm))
      return LSA_ERR_INVALID_ARG;
  }
  return LSA_OK;
}

extern "C" size_t lsa_state_size(void) { return sizeof(lsa_state); }
