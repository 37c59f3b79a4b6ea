// si_select_h32.cu -- the select kernel's instantiations for H_I = 32 (d_I 64
// and 128, pools in shared or global memory), in their own translation unit
// so that the library's kernels compile in parallel.
#include "si_host.cuh"

namespace si_host {

si_status launch_select_h32(const SelectLaunch& a) {
    if (a.D == 128) return launch_select_t<32, 128>(a);
    if (a.D == 64) return launch_select_t<32, 64>(a);
    return SI_ERR_UNSUPPORTED;
}

}  // namespace si_host
