// Kernel selection of the v4attn library.
#include "common.cuh"
#include "tc_kernels.h"

namespace v4a {

int mqa_split_keys(const v4attn_layer_desc* d) {
  (void)d;
  return kSimtSplitKeys;
}

cudaError_t index_scores_dispatch(const IndexParams& P, cudaStream_t st) {
  if (index_tc_supported(P)) return launch_index_tc(P, st);
  return launch_index_scores(P, st);
}

cudaError_t mqa_dispatch(const MqaParams& P, cudaStream_t st) { return launch_mqa_simt(P, st); }

cudaError_t project_dispatch(const ProjectParams& P, cudaStream_t st) {
  return launch_project(P, st);
}

const char* build_info_string() {
  return "v4attn sm_100a: compress(simt) index(tcgen05 mxf4 | simt) topk(radix) mqa(simt) project(simt)";
}

}  // namespace v4a
