// abi.cu -- the entry points of the C ABI that launch nothing: status names,
// the version, and the workspace size every call can use.
#include "common.cuh"
#include "workspace.cuh"

using namespace dfl;

extern "C" const char* dflash2_status_string(int status) {
    switch (status) {
        case DFLASH2_OK: return "DFLASH2_OK";
        case DFLASH2_EINVAL: return "DFLASH2_EINVAL: null pointer or invalid scalar argument";
        case DFLASH2_EDTYPE: return "DFLASH2_EDTYPE: unsupported dtype";
        case DFLASH2_ESHAPE: return "DFLASH2_ESHAPE: size outside the supported range";
        case DFLASH2_EWORKSPACE: return "DFLASH2_EWORKSPACE: workspace missing, misaligned or too small";
        case DFLASH2_ECUDA: return "DFLASH2_ECUDA: a CUDA launch or memset failed";
        case DFLASH2_EALIGN: return "DFLASH2_EALIGN: pointer or stride misaligned";
        default: return "DFLASH2_UNKNOWN_STATUS";
    }
}

extern "C" int dflash2_version(void) { return (1 << 16) | 0; }

extern "C" size_t dflash2_workspace_bytes(int B, int G, int64_t V) {
    if (B < 0 || G < 1 || G >= DFLASH2_MAX_BLOCK || V < 1) return 0;
    const int64_t rows = (int64_t)B * G;
    // sized for fp32 (es = 4), whose chunks are the shorter: serves bf16 too
    size_t need = topk_layout(rows, V, 4).total;
    need = need > greedy_layout(B, G, V, 4).total ? need : greedy_layout(B, G, V, 4).total;
    need = need > sample_layout(B, G, V, 4).total ? need : sample_layout(B, G, V, 4).total;
    need = need > select_layout(B, G).total ? need : select_layout(B, G).total;
    need = need > trunc_layout(B, G, V, 4).total ? need : trunc_layout(B, G, V, 4).total;
    need = need > greedy_ee_layout(B, G, V, 4).total ? need : greedy_ee_layout(B, G, V, 4).total;
    return need;
}

unsigned dfl_errors_topk(int clear);
unsigned dfl_errors_verify(int clear);
unsigned dfl_errors_dynconv(int clear);
unsigned dfl_errors_select(int clear);
unsigned dfl_errors_trunc(int clear);
unsigned dfl_errors_select_tc(int clear);
unsigned dfl_errors_greedy_ee(int clear);

extern "C" unsigned dflash2_device_errors(int clear) {
    const unsigned f[7] = {dfl_errors_topk(clear),      dfl_errors_verify(clear),
                           dfl_errors_dynconv(clear),   dfl_errors_select(clear),
                           dfl_errors_trunc(clear),     dfl_errors_select_tc(clear),
                           dfl_errors_greedy_ee(clear)};
    unsigned v = 0;
    for (unsigned x : f) {
        if (x == 0xFFFFFFFFu) return 0xFFFFFFFFu;
        v |= x;
    }
    return v;
}
