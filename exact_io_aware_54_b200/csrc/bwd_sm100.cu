#include "fa_internal.h"
namespace fa {
fa_status launch_bwd(const BwdLaunch&, cudaStream_t) { return FA_ERR_UNSUPPORTED; }
}
