// Launch functions of the steps around the attention: the draft inputs (GPU
// anchor sampler and draft-block builder) and the DSpark training loss.
#pragma once

#include "dspark_internal.cuh"

namespace dspark {

// draft inputs: GPU anchor sampler and the draft block's ids, positions, labels,
// Markov predecessors and eval_mask
cudaError_t launch_sample_anchors(const uint8_t *loss_mask, int B, int S, int N, uint64_t seed, int32_t *anchors,
                                  uint8_t *keep, cudaStream_t st);
cudaError_t launch_build_draft_inputs(const int32_t *input_ids, const uint8_t *loss_mask, int B, int S, int N,
                                      const int32_t *anchors, const uint8_t *keep, int mask_id, int32_t *draft_ids,
                                      int32_t *position_ids, int32_t *labels, int32_t *prev_ids, uint8_t *eval_mask,
                                      cudaStream_t st);

// DSpark loss over the draft steps and its gradient (cluster kernel)
size_t loss_workspace_size(int R);
int loss_seg(int V);  // vocabulary elements per CTA of a row's cluster
cudaError_t launch_loss(int R, int V, const void *L, const void *T, const int32_t *labels, const float *conf,
                        const uint8_t *mask, float ce_alpha, float l1_alpha, float conf_alpha, float *out,
                        void *grad, float *grad_conf, void *ws, uint64_t wait_ns, cudaStream_t st);

}  // namespace dspark
