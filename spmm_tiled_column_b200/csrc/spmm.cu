// spmm.cu -- prefill SpMM (placeholder until the tcgen05 kernel is in place).
#include "spw_internal.cuh"

using namespace spw;

extern "C" {

uint64_t spw_spmm_workspace_bytes(const spw_format* hdr, int M) {
    (void)hdr;
    (void)M;
    return 0;
}

int spw_spmm(const spw_format* hdr, const void* d_buf, const uint16_t* d_X, int M, int ldx,
             uint16_t* d_Y, int ldy, void* d_ws, uint64_t ws_bytes, void* stream) {
    int rc = check_header(hdr);
    if (rc != SPW_OK) return rc;
    if (!d_buf || !d_X || !d_Y || M < 0) return SPW_ERR_INVALID_ARG;
    if (!ld_ok(ldx, (int)hdr->K, M) || !ld_ok(ldy, (int)hdr->N, M)) return SPW_ERR_INVALID_ARG;
    if (!aligned16(d_buf) || !aligned16(d_X) || !aligned16(d_Y)) return SPW_ERR_ALIGNMENT;
    (void)d_ws; (void)ws_bytes; (void)stream;
    return SPW_ERR_UNSUPPORTED;
}

}  // extern "C"
