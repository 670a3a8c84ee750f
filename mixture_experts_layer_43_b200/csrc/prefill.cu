// prefill.cu -- prefill regime: not built yet; every call reports UNSUPPORTED.
#include "prefill.cuh"

namespace moe {

struct PrefillState {
    int unused;
};

size_t prefill_tile_capacity(const moe_config_t*) { return 1; }
PrefillState* prefill_state_create(const moe_config_t&) { return new PrefillState{0}; }
void prefill_state_destroy(PrefillState* s) { delete s; }
moe_status_t prefill_route(PrefillState*, const moe_config_t&, const Workspace&,
                           const moe_weights_t*, const uint16_t*, int, float*, cudaStream_t, int,
                           int* launches) {
    *launches = 0;
    return MOE_ERR_UNSUPPORTED;
}
moe_status_t prefill_experts(PrefillState*, const moe_config_t&, const Workspace&,
                             const moe_weights_t*, const uint16_t*, int, float*, cudaStream_t, int,
                             int* launches) {
    *launches = 0;
    return MOE_ERR_UNSUPPORTED;
}

}  // namespace moe
