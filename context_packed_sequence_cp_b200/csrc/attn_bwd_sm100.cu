#include "kernels.h"
namespace thd {
int launch_bwd_sm100(int, int, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                     const BwdArgs&, int, int, cudaStream_t) {
    return -2;
}
}  // namespace thd
