// Placeholder for the tensor-core path until its kernels land.
#include "internal.h"

namespace mla {
bool sm100_decode_supported(const mla_dims&) { return false; }
bool sm100_append_supported(const mla_dims&, int) { return false; }
void sm100_layout(const mla_dims& d, int batch, int n_q, int64_t max_len, int splits, mla_ws_layout* L) {
    generic_layout(d, batch, n_q, max_len, splits, L);
}
int sm100_decode(const DecodeCall&, int*) { return MLA_ERR_UNSUPPORTED; }
int sm100_append(const AppendCall&, int*) { return MLA_ERR_UNSUPPORTED; }
}  // namespace mla
