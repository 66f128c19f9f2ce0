// Kernel selection between the tensor-core (tcgen05) paths and the CUDA-core
// paths of the v4attn library (internal).
#pragma once

#include "../../include/v4attn.h"
#include "kernels.h"

namespace v4a {

// Keys per split-K chunk of the MQA kernel that serves this layer.
int mqa_split_keys(const v4attn_layer_desc* d);
// Split-K chunks per query for at most n_main_max entries per query (the
// entry and window key ranges are each padded to whole 64-key tiles).
int mqa_num_splits(const v4attn_layer_desc* d, int64_t n_main_max);

cudaError_t index_scores_dispatch(const IndexParams& P, cudaStream_t st);
cudaError_t mqa_dispatch(const MqaParams& P, cudaStream_t st);
cudaError_t project_dispatch(const ProjectParams& P, cudaStream_t st);
const char* build_info_string();

// 0: the tensor-core kernel takes these arguments; 1: a pointer is not
// 16-byte aligned; 2: a shape or format the kernel does not cover.
int index_tc_check(const IndexParams& P);
bool topk_cluster_supported(const TopkParams& P);
cudaError_t launch_topk_cluster(const TopkParams& P, cudaStream_t st);
cudaError_t topk_dispatch(const TopkParams& P, cudaStream_t st);
int mqa_tc_check(const MqaParams& P);   // as index_tc_check
int project_tc_check(const ProjectParams& P);   // as index_tc_check
cudaError_t launch_project_tc(const ProjectParams& P, cudaStream_t st);
// the driver's cuTensorMapEncodeTiled (nullptr when the driver lacks it)
void* tensor_map_encoder();
cudaError_t launch_mqa_tc(const MqaParams& P, cudaStream_t st);
cudaError_t launch_index_tc(const IndexParams& P, cudaStream_t st);

}  // namespace v4a
