// pa_api.cu -- small host-only entry points of the C ABI.
#include "pa.h"

extern "C" const char* pa_status_string(pa_status status)
{
    switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    }
    return "PA_ERR_UNKNOWN";
}

extern "C" const char* pa_version(void) { return "0.1.0"; }
