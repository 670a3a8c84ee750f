// prefill.cuh -- prefill-regime (T > MOE_DECODE_MAX_T, bf16) launch interface.
#pragma once

#include "moe_internal.cuh"

namespace moe {

struct PrefillState;

size_t prefill_tile_capacity(const moe_config_t* cfg);
PrefillState* prefill_state_create(const moe_config_t& cfg);
void prefill_state_destroy(PrefillState* s);
moe_status_t prefill_route(PrefillState* s, const moe_config_t& cfg, const Workspace& ws,
                           const moe_weights_t* w, const uint16_t* x, int T, float* out,
                           cudaStream_t stream, int num_sms, int* launches);
moe_status_t prefill_experts(PrefillState* s, const moe_config_t& cfg, const Workspace& ws,
                             const moe_weights_t* w, const uint16_t* x, int T, float* out,
                             cudaStream_t stream, int num_sms, int* launches);

}  // namespace moe
