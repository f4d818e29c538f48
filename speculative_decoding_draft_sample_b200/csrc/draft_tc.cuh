// Internal interface of the tensor-core (tcgen05) draft-logit kernel.
#pragma once

#include "draft.cuh"

namespace dspark {

// True when the tcgen05 path handles this shape (bf16, r % 16 == 0, r <= 256)
// and the driver's tensor-map encoder is reachable.
bool draft_tc_supported(const DraftArgs& a);
// Draft logits and chunk partials of position k (1-based), persistent CTAs.
cudaError_t draft_logits_tc_launch(const DraftArgs& a, int k, int num_sms, cudaStream_t s);
// True when all K positions fit one cooperative launch (M-tiles <= SMs).
bool draft_round_tc_supported(const DraftArgs& a, int num_sms);
// All K positions in one cooperative launch: logits, partials and the draw of
// every position, with grid barriers between them.
cudaError_t draft_round_tc_launch(const DraftArgs& a, int num_sms, cudaStream_t s);

}  // namespace dspark
