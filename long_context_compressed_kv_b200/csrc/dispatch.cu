// Kernel selection of the v4attn library.
#include "common.cuh"
#include "tc_kernels.h"

namespace v4a {

int mqa_split_keys(const v4attn_layer_desc* d) {
  if (d->kv_dtype == V4A_E4M3_BF16ROPE && d->d == 512)      // tensor-core kernel
    return d->kind == V4A_CSA ? 128 : 512;
  return kSimtSplitKeys;
}

int mqa_num_splits(const v4attn_layer_desc* d, int64_t n_main_max) {
  const int64_t pad = 64;
  const int64_t keys = (n_main_max + pad - 1) / pad * pad + (d->n_win + pad - 1) / pad * pad;
  const int sk = mqa_split_keys(d);
  return (int)std::max<int64_t>(1, (keys + sk - 1) / sk);
}

// MXFP4 runs on the tensor-core kernel only, F32 on CUDA cores only; the
// C-ABI has refused any MXFP4 call the tensor-core kernel does not take.
cudaError_t index_scores_dispatch(const IndexParams& P, cudaStream_t st) {
  if (P.idx_dtype == V4A_MXFP4)
    return index_tc_check(P) == 0 ? launch_index_tc(P, st) : cudaErrorNotSupported;
  return launch_index_scores(P, st);
}

cudaError_t topk_dispatch(const TopkParams& P, cudaStream_t st) {
  if (topk_cluster_supported(P)) return launch_topk_cluster(P, st);
  return launch_topk(P, st);
}

// E4M3 caches run on the tensor-core kernel only, F32 caches on CUDA cores.
cudaError_t mqa_dispatch(const MqaParams& P, cudaStream_t st) {
  if (P.kv_dtype == V4A_E4M3_BF16ROPE)
    return mqa_tc_check(P) == 0 ? launch_mqa_tc(P, st) : cudaErrorNotSupported;
  return launch_mqa_simt(P, st);
}

// bf16 projections run on the tensor-core GEMM only, fp32 ones on CUDA cores.
cudaError_t project_dispatch(const ProjectParams& P, cudaStream_t st) {
  if (P.x_dtype == V4A_BF16)
    return project_tc_check(P) == 0 ? launch_project_tc(P, st) : cudaErrorNotSupported;
  return launch_project(P, st);
}

const char* build_info_string() {
  return "v4attn sm_100a: compress(simt) index(mxfp4: tcgen05 mxf4; f32: simt) topk(cluster radix | radix) mqa(e4m3: tcgen05 fp8/bf16; f32: simt) project(bf16: tcgen05 f16; f32: simt)";
}

}  // namespace v4a
