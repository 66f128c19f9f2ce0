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

bool index_tc_supported(const IndexParams& P);
bool topk_cluster_supported(const TopkParams& P);
cudaError_t launch_topk_cluster(const TopkParams& P, cudaStream_t st);
cudaError_t topk_dispatch(const TopkParams& P, cudaStream_t st);
bool mqa_tc_supported(const MqaParams& P);
cudaError_t launch_mqa_tc(const MqaParams& P, cudaStream_t st);
cudaError_t launch_index_tc(const IndexParams& P, cudaStream_t st);

}  // namespace v4a
