// stubs.cu -- entry points of include/lka.h whose kernels are not part of this
// build yet: they validate nothing and report LKA_ERR_UNSUPPORTED.
#include "host_util.h"

extern "C" {

size_t latent_expand_gqa_attn_workspace_size(int, int, int, int, int, int, int) { return 0; }
lka_status_t latent_expand_gqa_attn(const void*, const void*, const void*, const void*, const void*,
                                    const int32_t*, void*, float*, int, int, int, int, int, int, int, int, float,
                                    lka_dtype_t, void*, size_t, void*) {
    return LKA_ERR_UNSUPPORTED;
}
size_t gta_shared_score_attn_workspace_size(int, int, int, int, int, int, int) { return 0; }
lka_status_t gta_shared_score_attn(const void*, const void*, const void*, const int32_t*, void*, float*, int, int,
                                   int, int, int, int, int, int, float, lka_dtype_t, void*, size_t, void*) {
    return LKA_ERR_UNSUPPORTED;
}

}  // extern "C"
