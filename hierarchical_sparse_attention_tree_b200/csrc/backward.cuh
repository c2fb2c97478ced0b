// Arguments of the decode-backward kernels, shared by their launchers and
// the C ABI's host code.
#pragma once

#include "common.cuh"

namespace recsa {

constexpr int PLAN_INTS = 72;          // valid, J, items, pad, then off[j], nc[j] for j = 0..MAXJ

struct BwdArgs {
    const void* q;     // [B][Hq][D], storage type
    const void* dout;  // [B][Hq][D], storage type (fp32 if dout_f32)
    const int* sel;    // [B*H][J_cap][k], the forward's selections
    float* dq;         // [B][Hq][D]
    float* dk;         // token gradients, the cache's row layout, [rows][D] (null: not wanted, with dv)
    float* dv;
    float* dw;         // [D][D], dW[r][c] for W[r][c]
    float* gK[MAXJ + 1];  // node-key gradient accumulators [B*H][rows[j]][D] (j >= 1)
    float* gV[MAXJ + 1];  // node-value gradient accumulators
    float* gW[MAXJ + 1];  // W^T h per node of levels 2..J_cap (the tree pass writes, then reads it)
    int* plan;         // [B*H][PLAN_INTS]
    int* ubase;        // [B*H + 1] first item of each unit in the list of all units' items
    float* lg;         // [B*H][E_cap][G] logits (-inf: not an entry)
    float* ag;         // [B*H][E_cap][G] <dout_g, v_e>
    float* st;         // [B*H][G][3] softmax maximum, denominator, sum_e p_e <dout, v_e>
    int E_cap;
    int dout_f32;
};

template <typename T, int D, int G>
cudaError_t launch_decode_backward(const TreeParams& p, const BwdArgs& a, cudaStream_t s);
template <typename T, int D>
cudaError_t launch_tree_backward(const TreeParams& p, const BwdArgs& a, long long max_len, cudaStream_t s);

}  // namespace recsa
