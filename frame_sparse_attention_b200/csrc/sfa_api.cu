// Status strings and version of libsfa.
#include "sfa.h"

extern "C" const char *sfa_error_string(sfa_status s)
{
    switch (s) {
    case SFA_OK: return "SFA_OK";
    case SFA_ERR_INVALID_ARG: return "SFA_ERR_INVALID_ARG: argument out of range";
    case SFA_ERR_UNSUPPORTED: return "SFA_ERR_UNSUPPORTED: valid but not implemented by this build";
    case SFA_ERR_CUDA: return "SFA_ERR_CUDA: a CUDA call or kernel launch failed";
    case SFA_ERR_TIMEOUT: return "SFA_ERR_TIMEOUT: a device pipeline wait reached its limit";
    case SFA_ERR_BAD_SET: return "SFA_ERR_BAD_SET: malformed attended-frame list on the device";
    }
    return "unknown sfa_status";
}

extern "C" int32_t sfa_version(void) { return 100; }
