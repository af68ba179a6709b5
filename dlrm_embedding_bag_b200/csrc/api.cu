// C ABI of the DLRMv1 sparse/interaction stage (declared in dlrm_sparse.h):
// host-side argument checks, packing of the table pointers into the kernel
// parameter block, and the launches. Nothing here allocates memory.
#include <climits>
#include <cstdint>
#include <cstring>

#include "dlrm_sparse.h"
#include "launch.h"

namespace dlrm {

thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return DLRM_ERR_CUDA;
}

}  // namespace dlrm

namespace {

using dlrm::cuda_fail;
using dlrm::t_last_cuda_error;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-block opt-in shared-memory limit of the current device.
int64_t smem_limit_current_device(int* err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = cuda_fail(e);
    return 0;
  }
  int v = 0;
  e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) {
    *err = cuda_fail(e);
    return 0;
  }
  *err = DLRM_OK;
  return v;
}

// A checked set of gather arguments, ready to launch.
struct Prepared {
  dlrm::TableParams tp;
  dlrm::BagParams bp;
  int pool;
  bool tables_aligned16;
  int elem_size;
};

// Checks shared by every gather entry point; fills the parameter blocks.
int prepare(const void* const* weights, int dtype, const int64_t* rows, const dlrm_bags_t* bags,
            int B, int F, int D, int32_t* status_dev, Prepared* pr) {
  if (bags == nullptr) return DLRM_ERR_NULL;
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  if (B < 1 || D < 1 || bags->T < 0 || bags->T > INT32_MAX) return DLRM_ERR_SHAPE;
  if (dtype != DLRM_TABLE_F32 && dtype != DLRM_TABLE_BF16) return DLRM_ERR_ARG;
  if (bags->mode != DLRM_POOL_SUM && bags->mode != DLRM_POOL_MEAN && bags->mode != DLRM_POOL_MAX)
    return DLRM_ERR_ARG;
  if (bags->per_sample_weights != nullptr && bags->mode != DLRM_POOL_SUM) return DLRM_ERR_ARG;
  if (weights == nullptr || bags->offsets == nullptr) return DLRM_ERR_NULL;
  if (bags->T > 0 && bags->indices == nullptr) return DLRM_ERR_NULL;
  if (!aligned(bags->offsets, 4) || (bags->indices && !aligned(bags->indices, 4)) ||
      (bags->per_sample_weights && !aligned(bags->per_sample_weights, 4)) ||
      (status_dev && !aligned(status_dev, 4)))
    return DLRM_ERR_ALIGN;
  const int esz = dtype == DLRM_TABLE_BF16 ? 2 : 4;
  std::memset(&pr->tp, 0, sizeof(pr->tp));
  bool a16 = true;
  for (int k = 0; k < F; ++k) {
    if (weights[k] == nullptr) return DLRM_ERR_NULL;
    if (!aligned(weights[k], esz)) return DLRM_ERR_ALIGN;
    a16 = a16 && aligned(weights[k], 16);
    pr->tp.w[k] = weights[k];
    if (rows != nullptr) {
      if (rows[k] < 0) return DLRM_ERR_ARG;
      pr->tp.rows[k] = rows[k] > INT32_MAX ? INT32_MAX : static_cast<int32_t>(rows[k]);
    }
  }
  pr->bp.indices = bags->indices;
  pr->bp.offsets = bags->offsets;
  pr->bp.psw = bags->per_sample_weights;
  pr->bp.T = static_cast<int>(bags->T);
  pr->bp.ilo = bags->include_last_offset ? 1 : 0;
  pr->bp.mean = bags->mode == DLRM_POOL_MEAN ? 1 : 0;
  pr->bp.check = rows != nullptr ? 1 : 0;
  pr->bp.status = status_dev;
  pr->bp.balance = 0;
  pr->pool = bags->per_sample_weights ? dlrm::kPoolWeighted
             : bags->mode == DLRM_POOL_MAX ? dlrm::kPoolMax
                                          : dlrm::kPoolSum;
  pr->tables_aligned16 = a16;
  pr->elem_size = esz;
  return DLRM_OK;
}

// The vector loader needs whole 16-byte chunks per row and 16-byte aligned
// tables and float destinations. f32 rows of at most 64 floats stream past L1
// (measured faster there; longer rows under skew gain from L1).
int pick_loader(int dtype, int D, bool vec_ok) {
  if (dtype == DLRM_TABLE_BF16)
    return (vec_ok && D % 8 == 0) ? dlrm::kLdBF16x8 : dlrm::kLdBF16x1;
  if (!vec_ok || D % 4 != 0) return dlrm::kLdF32x1;
  return D <= 64 ? dlrm::kLdF32x4S : dlrm::kLdF32x4;  // see LdF32x4S
}

int clear_status(int32_t* status_dev, cudaStream_t stream) {
  if (status_dev == nullptr) return DLRM_OK;
  cudaError_t e = cudaMemsetAsync(status_dev, 0, sizeof(int32_t), stream);
  return e == cudaSuccess ? DLRM_OK : cuda_fail(e);
}

dlrm::GatherPlan make_plan(const Prepared& pr, int B, int F, int D, int loader) {
  dlrm::GatherPlan g;
  g.tp = &pr.tp;
  g.bp = pr.bp;
  g.B = B;
  g.F = F;
  g.D = D;
  g.pool = pr.pool;
  g.loader = loader;
  g.esz = pr.elem_size;
  return g;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? DLRM_OK : cuda_fail(e); }

int pool_impl(const void* const* weights, int dtype, const int64_t* rows, const dlrm_bags_t* bags,
              int B, int F, int D, float* out, int32_t* status_dev, cudaStream_t stream) {
  Prepared pr;
  int rc = prepare(weights, dtype, rows, bags, B, F, D, status_dev, &pr);
  if (rc != DLRM_OK) return rc;
  if (out == nullptr) return DLRM_ERR_NULL;
  if (!aligned(out, 4)) return DLRM_ERR_ALIGN;
  const bool out16 = aligned(out, 16);
  const int loader = pick_loader(dtype, D, pr.tables_aligned16 && out16);
  const dlrm::GatherPlan g = make_plan(pr, B, F, D, loader);
  if ((rc = clear_status(status_dev, stream)) != DLRM_OK) return rc;
  return launch_status(dlrm::launch_embbag(g, out, stream));
}

int fused_impl(const void* const* weights, int dtype, const int64_t* rows,
               const dlrm_bags_t* bags, const float* dense, int B, int F, int D,
               float* pooled_out, float* inter_out, int concat_dense, int32_t* status_dev,
               bool fixed_stride, cudaStream_t stream) {
  Prepared pr;
  int rc = prepare(weights, dtype, rows, bags, B, F, D, status_dev, &pr);
  if (rc != DLRM_OK) return rc;
  // bags of any lengths: the fused kernel orders each block's bags by length
  pr.bp.balance = fixed_stride ? 0 : 1;
  if (dense == nullptr || inter_out == nullptr) return DLRM_ERR_NULL;
  if (!aligned(dense, 4) || !aligned(inter_out, 4) || (pooled_out && !aligned(pooled_out, 4)))
    return DLRM_ERR_ALIGN;
  int err = DLRM_OK;
  const int64_t limit = smem_limit_current_device(&err);
  if (err != DLRM_OK) return err;
  if (dlrm::interact_smem_per_sample(F, D) > limit) return DLRM_ERR_SHAPE;
  const bool pooled16 = pooled_out == nullptr || aligned(pooled_out, 16);
  const int loader = pick_loader(dtype, D, pr.tables_aligned16 && pooled16);
  const dlrm::GatherPlan g = make_plan(pr, B, F, D, loader);
  if ((rc = clear_status(status_dev, stream)) != DLRM_OK) return rc;
  return launch_status(dlrm::launch_fused(g, dense, pooled_out, inter_out, concat_dense ? 1 : 0,
                                          limit, stream));
}

// The fixed-stride, unweighted-sum, f32 case of the general entry points.
int fixed_stride_bags(const int32_t* indices, const int32_t* offsets, int B, int L,
                      dlrm_bags_t* bags) {
  if (B < 1 || L < 0) return DLRM_ERR_SHAPE;
  if (static_cast<int64_t>(B) * L > INT32_MAX) return DLRM_ERR_SHAPE;
  bags->indices = indices;
  bags->offsets = offsets;
  bags->per_sample_weights = nullptr;
  bags->T = static_cast<int64_t>(B) * L;
  bags->include_last_offset = 0;
  bags->mode = DLRM_POOL_SUM;
  return DLRM_OK;
}

const void* const* as_void(const float* const* w) {
  return reinterpret_cast<const void* const*>(w);
}

}  // namespace

extern "C" {

int embbag_sum_multi(const float* const* weights, const int32_t* indices, const int32_t* offsets,
                     int B, int F, int L, int D, float* out, dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  dlrm_bags_t bags;
  int rc = fixed_stride_bags(indices, offsets, B, L, &bags);
  if (rc != DLRM_OK) return rc;
  return pool_impl(as_void(weights), DLRM_TABLE_F32, nullptr, &bags, B, F, D, out, nullptr,
                   reinterpret_cast<cudaStream_t>(stream));
}

int embbag_sum_multi_ex(const float* const* weights, const int64_t* rows, const int32_t* indices,
                        const int32_t* offsets, int B, int F, int L, int D, float* out,
                        int32_t* status_dev, dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  if (rows == nullptr) return DLRM_ERR_NULL;
  dlrm_bags_t bags;
  int rc = fixed_stride_bags(indices, offsets, B, L, &bags);
  if (rc != DLRM_OK) return rc;
  return pool_impl(as_void(weights), DLRM_TABLE_F32, rows, &bags, B, F, D, out, status_dev,
                   reinterpret_cast<cudaStream_t>(stream));
}

int embbag_pool_multi(const void* const* weights, int table_dtype, const int64_t* rows,
                      const dlrm_bags_t* bags, int B, int F, int D, float* out,
                      int32_t* status_dev, dlrm_stream_t stream) {
  return pool_impl(weights, table_dtype, rows, bags, B, F, D, out, status_dev,
                   reinterpret_cast<cudaStream_t>(stream));
}

int interact_lower_tri(const float* dense, const float* emb, int B, int F, int D, float* out,
                       dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  if (B < 1 || D < 1) return DLRM_ERR_SHAPE;
  if (dense == nullptr || emb == nullptr || out == nullptr) return DLRM_ERR_NULL;
  if (!aligned(dense, 4) || !aligned(emb, 4) || !aligned(out, 4)) return DLRM_ERR_ALIGN;
  int err = DLRM_OK;
  const int64_t limit = smem_limit_current_device(&err);
  if (err != DLRM_OK) return err;
  if (dlrm::interact_smem_per_sample(F, D) > limit) return DLRM_ERR_SHAPE;
  const bool vec_ok = (D % 4 == 0) && aligned(dense, 16) && aligned(emb, 16);
  cudaError_t e = dlrm::launch_interact(dense, emb, B, F, D, out, vec_ok, limit,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DLRM_OK : cuda_fail(e);
}

int dlrm_sparse_interact(const float* const* weights, const int32_t* indices,
                         const int32_t* offsets, const float* dense, int B, int F, int L, int D,
                         float* pooled_out, float* inter_out, int concat_dense,
                         dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  dlrm_bags_t bags;
  int rc = fixed_stride_bags(indices, offsets, B, L, &bags);
  if (rc != DLRM_OK) return rc;
  return fused_impl(as_void(weights), DLRM_TABLE_F32, nullptr, &bags, dense, B, F, D,
                    pooled_out, inter_out, concat_dense, nullptr, true,
                    reinterpret_cast<cudaStream_t>(stream));
}

int dlrm_sparse_interact_ex(const float* const* weights, const int64_t* rows,
                            const int32_t* indices, const int32_t* offsets, const float* dense,
                            int B, int F, int L, int D, float* pooled_out, float* inter_out,
                            int concat_dense, int32_t* status_dev, dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  if (rows == nullptr) return DLRM_ERR_NULL;
  dlrm_bags_t bags;
  int rc = fixed_stride_bags(indices, offsets, B, L, &bags);
  if (rc != DLRM_OK) return rc;
  return fused_impl(as_void(weights), DLRM_TABLE_F32, rows, &bags, dense, B, F, D, pooled_out,
                    inter_out, concat_dense, status_dev, true,
                    reinterpret_cast<cudaStream_t>(stream));
}

int dlrm_sparse_interact_pool(const void* const* weights, int table_dtype, const int64_t* rows,
                              const dlrm_bags_t* bags, const float* dense, int B, int F, int D,
                              float* pooled_out, float* inter_out, int concat_dense,
                              int32_t* status_dev, dlrm_stream_t stream) {
  return fused_impl(weights, table_dtype, rows, bags, dense, B, F, D, pooled_out, inter_out,
                    concat_dense, status_dev, false, reinterpret_cast<cudaStream_t>(stream));
}

int dlrm_sparse_interact_host(const float* const* weights, const int32_t* indices_host,
                              const int32_t* offsets_host, const float* dense_host, int B, int F,
                              int L, int D, int concat_dense, int32_t* indices_dev,
                              int32_t* offsets_dev, float* dense_dev, float* pooled_dev,
                              float* inter_dev, float* pooled_host, float* inter_host,
                              dlrm_stream_t stream) {
  if (F < 1 || F > DLRM_MAX_TABLES) return DLRM_ERR_TOO_MANY_TABLES;
  if (B < 1 || L < 0 || D < 1) return DLRM_ERR_SHAPE;
  if (static_cast<int64_t>(B) * L > INT32_MAX) return DLRM_ERR_SHAPE;
  if (offsets_host == nullptr || dense_host == nullptr || inter_host == nullptr ||
      offsets_dev == nullptr || dense_dev == nullptr || inter_dev == nullptr)
    return DLRM_ERR_NULL;
  if (L > 0 && (indices_host == nullptr || indices_dev == nullptr)) return DLRM_ERR_NULL;
  if (pooled_host != nullptr && pooled_dev == nullptr) return DLRM_ERR_NULL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t P = static_cast<int64_t>(F + 1) * F / 2;
  const size_t n_idx = static_cast<size_t>(F) * B * L * sizeof(int32_t);
  const size_t n_off = static_cast<size_t>(F) * B * sizeof(int32_t);
  const size_t n_dense = static_cast<size_t>(B) * D * sizeof(float);
  const size_t n_inter = static_cast<size_t>(B) * (concat_dense ? D + P : P) * sizeof(float);
  const size_t n_pooled = static_cast<size_t>(B) * F * D * sizeof(float);
  cudaError_t e;
  // indices, offsets and dense back to back on both sides (no gap): one copy
  const auto* ih = reinterpret_cast<const char*>(indices_host);
  auto* id = reinterpret_cast<char*>(indices_dev);
  const bool packed = n_idx > 0 &&
                      reinterpret_cast<const char*>(offsets_host) == ih + n_idx &&
                      reinterpret_cast<const char*>(dense_host) == ih + n_idx + n_off &&
                      reinterpret_cast<char*>(offsets_dev) == id + n_idx &&
                      reinterpret_cast<char*>(dense_dev) == id + n_idx + n_off;
  if (packed) {
    if ((e = cudaMemcpyAsync(id, ih, n_idx + n_off + n_dense, cudaMemcpyHostToDevice, s)) !=
        cudaSuccess)
      return cuda_fail(e);
  } else {
    if (n_idx > 0 &&
        (e = cudaMemcpyAsync(indices_dev, indices_host, n_idx, cudaMemcpyHostToDevice, s)) !=
            cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaMemcpyAsync(offsets_dev, offsets_host, n_off, cudaMemcpyHostToDevice, s)) !=
        cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaMemcpyAsync(dense_dev, dense_host, n_dense, cudaMemcpyHostToDevice, s)) !=
        cudaSuccess)
      return cuda_fail(e);
  }
  int rc = dlrm_sparse_interact(weights, indices_dev, offsets_dev, dense_dev, B, F, L, D,
                                pooled_dev, inter_dev, concat_dense, stream);
  if (rc != DLRM_OK) return rc;
  if ((e = cudaMemcpyAsync(inter_host, inter_dev, n_inter, cudaMemcpyDeviceToHost, s)) !=
      cudaSuccess)
    return cuda_fail(e);
  if (pooled_host &&
      (e = cudaMemcpyAsync(pooled_host, pooled_dev, n_pooled, cudaMemcpyDeviceToHost, s)) !=
          cudaSuccess)
    return cuda_fail(e);
  return DLRM_OK;
}

int dlrm_pair_decode(int64_t p0, int64_t count, int32_t* i_out, int32_t* j_out,
                     dlrm_stream_t stream) {
  if (p0 < 0 || count < 0 || p0 + count > (int64_t{1} << 31)) return DLRM_ERR_ARG;
  if (count > 0 && (i_out == nullptr || j_out == nullptr)) return DLRM_ERR_NULL;
  if ((i_out && !aligned(i_out, 4)) || (j_out && !aligned(j_out, 4))) return DLRM_ERR_ALIGN;
  cudaError_t e =
      dlrm::launch_pair_decode(p0, count, i_out, j_out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DLRM_OK : cuda_fail(e);
}

int dlrm_set_gather_path(int path) {
  if (path != DLRM_PATH_AUTO && path != DLRM_PATH_LDG) return DLRM_ERR_ARG;
  const int prev = dlrm::gather_path();
  dlrm::set_gather_path(path);
  return prev;
}

int dlrm_last_gather_path(void) { return dlrm::last_path(); }

int dlrm_status_from_flags(int32_t flags) {
  if (flags & DLRM_FLAG_TIMEOUT) return DLRM_ERR_TIMEOUT;
  if (flags & DLRM_FLAG_INDEX_OOB) return DLRM_ERR_INDEX_OOB;
  if (flags & DLRM_FLAG_OFFSETS) return DLRM_ERR_OFFSETS;
  return DLRM_OK;
}

const char* dlrm_status_string(int status) {
  switch (status) {
    case DLRM_OK: return "ok";
    case DLRM_ERR_NULL: return "a required pointer is NULL";
    case DLRM_ERR_SHAPE: return "invalid shape (B, L, D, T, or shared memory needed per sample)";
    case DLRM_ERR_ALIGN: return "a pointer is not aligned to its element size";
    case DLRM_ERR_TOO_MANY_TABLES: return "table count F must be in [1, DLRM_MAX_TABLES]";
    case DLRM_ERR_INDEX_OOB: return "an index lies outside its table";
    case DLRM_ERR_OFFSETS: return "offsets describe a bag with start > end or outside [0, T]";
    case DLRM_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case DLRM_ERR_ARG: return "invalid argument";
    case DLRM_ERR_TIMEOUT: return "a bounded wait on an asynchronous copy ran out";
    case DLRM_ERR_SCRATCH:
      return "the call needs more device staging than the library's fixed array holds";
    default: return "unknown status";
  }
}

int dlrm_last_cuda_error(void) { return t_last_cuda_error; }

int64_t dlrm_launch_count(void) { return dlrm::launch_count(); }

int dlrm_probe_bounded_wait(int64_t limit_cycles, int32_t* status_dev, dlrm_stream_t stream) {
  if (status_dev == nullptr) return DLRM_ERR_NULL;
  if (!aligned(status_dev, 4)) return DLRM_ERR_ALIGN;
  const int64_t limit =
      limit_cycles < 1000 ? 1000 : (limit_cycles > 200000000 ? 200000000 : limit_cycles);
  const cudaError_t e =
      dlrm::launch_probe_wait(limit, status_dev, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DLRM_OK : cuda_fail(e);
}

int dlrm_probe_row_gather(const void* table, int64_t rows, int row_bytes, int64_t count,
                          uint64_t seed, uint32_t* sink_dev, dlrm_stream_t stream) {
  if (table == nullptr || sink_dev == nullptr) return DLRM_ERR_NULL;
  if (row_bytes != 16 && row_bytes != 32 && row_bytes != 64 && row_bytes != 128 &&
      row_bytes != 256 && row_bytes != 512)
    return DLRM_ERR_SHAPE;
  if (rows < 1 || count < 0) return DLRM_ERR_SHAPE;
  if (!aligned(table, 16) || !aligned(sink_dev, 4)) return DLRM_ERR_ALIGN;
  const cudaError_t e = dlrm::launch_probe_row_gather(
      table, rows, row_bytes / 16, count, seed, sink_dev, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DLRM_OK : cuda_fail(e);
}

}  // extern "C"
