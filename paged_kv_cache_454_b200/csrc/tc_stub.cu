// Placeholder for the tcgen05 kernels (not built yet): reports them unsupported.
#include "internal.h"
namespace pa {
bool decode_tcgen05_supported(int, int) { return false; }
bool prefill_tcgen05_supported(const PrefillArgs&) { return false; }
int launch_decode_tcgen05(const DecodeArgs&) { return PA_ERR_UNSUPPORTED; }
int launch_prefill_tcgen05(const PrefillArgs&) { return PA_ERR_UNSUPPORTED; }
}  // namespace pa
