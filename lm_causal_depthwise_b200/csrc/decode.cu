// decode.cu -- batched single-token step (bf16).
#include "internal.h"

namespace rglru {

size_t decode_workspace_bytes(int B, int D) { return simt_workspace_bytes(B, 1, D); }

rglru_status decode_step(const PrefillArgs &a) { return simt_prefill(a); }

}  // namespace rglru
