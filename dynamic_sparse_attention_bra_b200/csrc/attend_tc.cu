#include "attend_tc.h"

namespace bra {

bra_status attend_tc_launch(const Geometry&, const void*, const void*, const void*,
                            const int32_t*, void*, int*, cudaStream_t) {
    return BRA_ERR_UNSUPPORTED;
}

}  // namespace bra
