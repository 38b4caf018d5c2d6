// prefill_fused.cu -- bf16 prefill entry (fused sm_100a kernel goes here).
#include "internal.h"

namespace rglru {

size_t fused_workspace_bytes(int B, int T, int D) { return simt_workspace_bytes(B, T, D); }

rglru_status fused_prefill(const PrefillArgs &a) { return simt_prefill(a); }

}  // namespace rglru
