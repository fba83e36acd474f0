// spmv_auto.cu -- decode with the path chosen by batch size.
//
// "Unified Static-Dynamic Pruning for Efficient LLM Inference" (abstract) calls the
// bitmap decoding of its spMspV kernel "hybrid" without saying between what; this
// library reads it as a runtime choice between its two decode paths, taken per call from
// the batch size:
//   - spw_spmv (CUDA cores): every kept weight costs B multiply-adds per lane, so its
//     time grows with the batch;
//   - spw_spmv_tc (tensor cores): the decoded weight tile is the MMA's A operand and the
//     batch its N, so its time hardly changes from B = 4 to 16.
// Measured on one B200 (graph-timed over rotated copies, 50 % sparsity, dense input), us
// per call, CUDA-core / tensor-core:
//   B                 4            8            12           14           16
//   q 4096x4096       18.2 / 29.8  30.1 / 29.8  34.6 / 29.8  39.9 / 29.9  40.2 / 29.9
//   gate 11008x4096   27.7 / 73.9  42.3 / 74.5  65.0 / 74.4  75.2 / 74.6  76.4 / 74.5
//   down 4096x11008   29.3 / 69.5  47.7 / 69.8  66.3 / 69.9  76.9 / 70.0  77.5 / 69.9
// The tensor-core time is flat in B and the CUDA-core time grows with it; from 14 rows
// the tensor-core path is the faster on every shape (the Llama-13B shapes agree at 16),
// below 12 rows the CUDA-core path is on the two large shapes.  The choice depends on B
// alone, so it is made on the host before the launch and needs no device read.
#include "spw_internal.cuh"

namespace {

constexpr int kTcMinBatch = 14;

bool takes_tensor_cores(int B) { return B >= kTcMinBatch; }

}  // namespace

extern "C" {

int spw_spmv_auto_path(int B) {
    if (B < 1 || B > 16) return -1;
    return takes_tensor_cores(B) ? 1 : 0;
}

uint64_t spw_spmv_auto_workspace_bytes(const spw_format* hdr, int B) {
    if (B < 1 || B > 16) return 0;
    return takes_tensor_cores(B) ? spw_spmv_tc_workspace_bytes(hdr, B) : spw_spmv_workspace_bytes(hdr, B);
}

int spw_spmv_auto(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B, int ldx,
                  float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy, void* d_ws,
                  uint64_t ws_bytes, void* stream) {
    if (B < 1 || B > 16) return SPW_ERR_INVALID_ARG;
    if (takes_tensor_cores(B))
        return spw_spmv_tc(hdr, d_buf, d_x, B, ldx, threshold, d_act_bits, d_y, ldy, d_ws, ws_bytes,
                           stream);
    return spw_spmv(hdr, d_buf, d_x, B, ldx, threshold, d_act_bits, d_y, ldy, d_ws, ws_bytes, stream);
}

}  // extern "C"
