// Decode step of the Gated DeltaNet mixer: one token for each of `rows` rows.
//
// Qwen3.8 27B model card (Nestmodels for Linnet), "Gated DeltaNet" bullet and
// cache paragraph: each row keeps its conv history and its per-value-head
// [128,128] f32 state; one token conv + silu, L2-normalised q and k, decay
// exp(g) with g = -exp(A_log) * softplus(a + dt_bias), write rate
// beta = sigmoid(b), the gated delta rule, and the gated RMSNorm of the read-out.
//
// The step is bound by HBM bandwidth: every row's state (48 x 64 KiB) is read
// and written once.  One CTA owns one (row, value head) state; each of its 8
// warps streams 16 state rows with 128-bit coalesced loads (a 128-float row is
// one 512-byte warp access), keeps them in registers, and forms S.k and S.q
// with warp-shuffle reductions.  Because
//     S_new = alpha S + u k^T,  u = beta (v - alpha S k),
//     o     = S_new q = alpha (S q) + u (k . q),
// both dot products use the old row, so each state row is read once and
// written once.
//
// The conv history of the q/k channels is shared by the value heads of one
// q/k head; those CTAs form one thread-block cluster, read the history first,
// and rewrite it only after a cluster barrier, so the in-place update is safe.
#pragma once

#include "common.cuh"

namespace gdn {

struct DecodeParams {
    int Kh, Vh, C, rows;
    const uint16_t* qkv;     // bf16 [rows][C]
    const uint16_t* z;       // bf16 [rows][Vh*128]
    const uint16_t* a;       // bf16 [rows][Vh]
    const uint16_t* b;       // bf16 [rows][Vh]
    const uint16_t* conv_w;  // bf16 [C][4]
    const float* A_log;      // [Vh]
    const float* dt_bias;    // [Vh]
    const float* norm_w;     // [128]
    float* state;            // f32 [rows][Vh][128][128], in place
    float* conv;             // f32 [rows][3][C], in place
    uint16_t* out;           // bf16 [rows][Vh*128]
};

constexpr int kDecThreads = 256;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__global__ void __launch_bounds__(kDecThreads, 2) gdn_decode_kernel(const DecodeParams p) {
    const int h = blockIdx.x;
    const int row = blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int group = p.Vh / p.Kh;
    const int kap = h / group;

    __shared__ float s_q[kD], s_k[kD], s_v[kD], s_o[kD];
    __shared__ float s_red[8];
    __shared__ float s_gate[2];

    // 1. Issue this warp's 16 state-row loads first; they are independent of
    //    the token's conv and gates and cover the HBM latency.
    float* Sbase = p.state + ((size_t)row * p.Vh + h) * kD * kD;
    float4 s[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
        s[r] = __ldcs(reinterpret_cast<const float4*>(Sbase + (size_t)(warp * 16 + r) * kD) + lane);

    // 2. Conv + silu for the q, k channels of q/k head kap and the v channels of head h.
    //    idx in [0,384): 0..127 q, 128..255 k, 256..383 v.  Thread tid handles tid and tid+256.
    float hist_keep[2][3];
    int ch_keep[2];
    bool write_keep[2];
    const unsigned int crank = (unsigned int)(h % group);  // rank inside the cluster of value heads
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int idx = tid + u * kDecThreads;
        ch_keep[u] = -1;
        write_keep[u] = false;
        if (idx >= 3 * kD) continue;
        const int grp = idx / kD, c = idx % kD;
        const int ch = (grp == 0) ? kap * kD + c : (grp == 1) ? p.Kh * kD + kap * kD + c : 2 * p.Kh * kD + h * kD + c;
        const float* hrow = p.conv + (size_t)row * 3 * p.C + ch;
        const float h0 = hrow[0], h1 = hrow[p.C], h2 = hrow[2 * p.C];
        const float x = bf16_bits_to_float(p.qkv[(size_t)row * p.C + ch]);
        const uint2 wbits = *reinterpret_cast<const uint2*>(p.conv_w + (size_t)ch * 4);
        const float w0 = __uint_as_float(wbits.x << 16), w1 = __uint_as_float(wbits.x & 0xffff0000u);
        const float w2 = __uint_as_float(wbits.y << 16), w3 = __uint_as_float(wbits.y & 0xffff0000u);
        const float cv = w0 * h0 + w1 * h1 + w2 * h2 + w3 * x;
        const float act = silu_f(cv);
        if (grp == 0) s_q[c] = act;
        else if (grp == 1) s_k[c] = act;
        else s_v[c] = act;
        hist_keep[u][0] = h1;
        hist_keep[u][1] = h2;
        hist_keep[u][2] = x;
        ch_keep[u] = ch;
        write_keep[u] = (grp == 2) || (crank == 0);
    }
    // All history reads of this CTA are done: let the cluster's other CTAs proceed to rewrite.
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");

    if (tid == 0) {
        const float av = bf16_bits_to_float(p.a[(size_t)row * p.Vh + h]);
        const float bv = bf16_bits_to_float(p.b[(size_t)row * p.Vh + h]);
        s_gate[0] = -expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
        s_gate[1] = sigmoid_f(bv);
    }
    __syncthreads();

    // 3. L2 norms of q (warps 0-3) and k (warps 4-7).
    {
        const float x = (tid < kD) ? s_q[tid] : s_k[tid - kD];
        const float ss = warp_sum(x * x);
        if (lane == 0) s_red[warp] = ss;
    }
    __syncthreads();
    const float qss = s_red[0] + s_red[1] + s_red[2] + s_red[3];
    const float kss = s_red[4] + s_red[5] + s_red[6] + s_red[7];
    const float qscale = rsqrtf(qss + kEps) * rsqrtf((float)kD);
    const float kscale = rsqrtf(kss + kEps);
    const float4 q4 = reinterpret_cast<const float4*>(s_q)[lane];
    const float4 k4 = reinterpret_cast<const float4*>(s_k)[lane];
    const float4 qf = make_float4(q4.x * qscale, q4.y * qscale, q4.z * qscale, q4.w * qscale);
    const float4 kf = make_float4(k4.x * kscale, k4.y * kscale, k4.z * kscale, k4.w * kscale);
    const float kq = warp_sum(kf.x * qf.x + kf.y * qf.y + kf.z * qf.z + kf.w * qf.w);
    const float alpha = expf(s_gate[0]);
    const float beta = s_gate[1];

    // 4. Stream the state rows: read once, update, write once.
#pragma unroll
    for (int r = 0; r < 16; ++r) {
        const int i = warp * 16 + r;
        const float dk = warp_sum(s[r].x * kf.x + s[r].y * kf.y + s[r].z * kf.z + s[r].w * kf.w);
        const float dq = warp_sum(s[r].x * qf.x + s[r].y * qf.y + s[r].z * qf.z + s[r].w * qf.w);
        const float u = beta * (s_v[i] - alpha * dk);
        float4 n;
        n.x = alpha * s[r].x + u * kf.x;
        n.y = alpha * s[r].y + u * kf.y;
        n.z = alpha * s[r].z + u * kf.z;
        n.w = alpha * s[r].w + u * kf.w;
        __stcs(reinterpret_cast<float4*>(Sbase + (size_t)i * kD) + lane, n);
        if (lane == 0) s_o[i] = alpha * dq + u * kq;
    }
    __syncthreads();

    // 5. Gated RMSNorm over the head's 128 outputs.
    {
        const float o = (tid < kD) ? s_o[tid] : 0.0f;
        const float ss = warp_sum(o * o);
        if (lane == 0) s_red[warp] = ss;
    }
    __syncthreads();
    if (tid < kD) {
        const float ms = (s_red[0] + s_red[1] + s_red[2] + s_red[3]) * (1.0f / kD);
        const float zval = bf16_bits_to_float(p.z[(size_t)row * p.Vh * kD + h * kD + tid]);
        const float y = s_o[tid] * rsqrtf(ms + kEps) * (1.0f + p.norm_w[tid]) * silu_f(zval);
        p.out[(size_t)row * p.Vh * kD + h * kD + tid] = float_to_bf16_bits(y);
    }

    // 6. History shift, after every CTA of the cluster has read the old values.
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        if (ch_keep[u] >= 0 && write_keep[u]) {
            float* hrow = p.conv + (size_t)row * 3 * p.C + ch_keep[u];
            hrow[0] = hist_keep[u][0];
            hrow[p.C] = hist_keep[u][1];
            hrow[2 * p.C] = hist_keep[u][2];
        }
    }
}

}  // namespace gdn
