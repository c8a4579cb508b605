// prefill.cu -- tcgen05 prefill kernel (not built yet: reports "not supported").
#include "internal.h"

namespace blasst {

cudaError_t launch_prefill(const PrefillParams &, const CUtensorMap &, const CUtensorMap &, const CUtensorMap &, bool,
                           cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace blasst
