// Placeholder for the tcgen05 prefill kernel (not built yet): reports it unsupported.
#include "internal.h"
namespace pa {
bool prefill_tcgen05_supported(const PrefillArgs&) { return false; }
int launch_prefill_tcgen05(const PrefillArgs&) { return PA_ERR_UNSUPPORTED; }
}  // namespace pa
