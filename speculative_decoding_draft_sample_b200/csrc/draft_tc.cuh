// Internal interface of the tensor-core (tcgen05) draft-logit kernel.
#pragma once

#include "draft.cuh"

namespace dspark {

// True when the tcgen05 path handles this shape (bf16, r % 16 == 0, r <= 256)
// and the driver's tensor-map encoder is reachable.
bool draft_tc_supported(const DraftArgs& a);
// Draft logits and chunk partials of position k (1-based), persistent CTAs.
cudaError_t draft_logits_tc_launch(const DraftArgs& a, int k, int num_sms, cudaStream_t s);
// SMs the one-launch draft leaves free unless the caller asks for more: room
// for the prefix schedule, which runs on another stream at the same time.
constexpr int kDraftFreeSms = 2;
// True when all K positions fit one cooperative launch (M-tiles <= SMs - kDraftFreeSms).
bool draft_round_tc_supported(const DraftArgs& a, int num_sms);
// All K positions in one cooperative launch: logits, partials and the draw of
// every position, with grid barriers between them. free_sms SMs stay free for
// work on other streams, clamped so that every M-tile keeps at least one CTA;
// the results do not depend on it (only the grid does).
cudaError_t draft_round_tc_launch(const DraftArgs& a, int num_sms, int free_sms, cudaStream_t s);

}  // namespace dspark
