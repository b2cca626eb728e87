// Status strings of the C ABI.
#include "gsa.h"

extern "C" const char* gsa_status_string(gsa_status status) {
    switch (status) {
        case GSA_OK: return "GSA_OK";
        case GSA_ERR_ARG: return "GSA_ERR_ARG: invalid argument (null pointer, k/W/chunk out of range, empty context)";
        case GSA_ERR_SHAPE: return "GSA_ERR_SHAPE: unsupported shape (head_dim, head grouping or size)";
        case GSA_ERR_DTYPE: return "GSA_ERR_DTYPE: unsupported element type";
        case GSA_ERR_ALIGN: return "GSA_ERR_ALIGN: tensor pointer not 16-byte aligned";
        case GSA_ERR_WORKSPACE: return "GSA_ERR_WORKSPACE: workspace missing, too small or misaligned";
        case GSA_ERR_CUDA: return "GSA_ERR_CUDA: a CUDA call or kernel launch failed";
        case GSA_ERR_TIMEOUT: return "GSA_ERR_TIMEOUT: a device-side bounded wait expired";
    }
    return "unknown gsa_status";
}
