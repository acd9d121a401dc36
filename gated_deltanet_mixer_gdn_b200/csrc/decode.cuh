// Decode step of the Gated DeltaNet mixer: one token for each of `rows` rows.
//
// Qwen3.8 27B model card (Nestmodels for Linnet), "Gated DeltaNet" bullet and
// cache paragraph: each row keeps its conv history and its per-value-head
// [128,128] f32 state; one token conv + silu, L2-normalised q and k, decay
// exp(g) with g = -exp(A_log) * softplus(a + dt_bias), write rate
// beta = sigmoid(b), the gated delta rule, and the gated RMSNorm of the read-out.
//
// The step is bound by HBM bandwidth: every row's state (48 x 64 KiB) is read
// and written once.  Because
//     S_new = alpha S + u k^T,  u = beta (v - alpha S k),
//     o     = S_new q = alpha (S q) + u (k . q),
// both dot products use the old state row, so each row is read and written
// once.
//
// Layout of the work: a persistent CTA owns one value head h and the rows
// p, p + P, p + 2P, ...  A producer warp streams the state in 32 KiB
// half-tiles (64 state rows) with bulk copies into a ring of shared-memory
// stages and writes each updated half-tile back with a bulk store; eight
// compute warps update a half-tile in shared memory, 8 state rows per warp,
// a 128-bit load per lane per row, with the 16 dot products of a warp reduced
// by one transposed shuffle reduction.  The conv / norm / gate prologue of the
// next row is prefetched into registers while the current row streams.
//
// The conv history of the q/k channels is shared by the value heads of one
// q/k head; those CTAs form one thread-block cluster (same rows), read the
// history first, and rewrite it only after a cluster barrier, so the in-place
// shift is safe.
#pragma once

#include "common.cuh"

namespace gdn {

struct DecodeParams {
    int Kh, Vh, C, rows, P;
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

#ifndef GDN_DECODE_STAGES
#define GDN_DECODE_STAGES 6
#endif
#ifndef GDN_DECODE_STORE_LAG
#define GDN_DECODE_STORE_LAG 1
#endif

namespace dec {
constexpr int kStages = GDN_DECODE_STAGES;
// A stage is refilled once the bulk store issued this many units later has
// been started, so a store has that long to drain before its stage is reused.
constexpr int kStoreLag = GDN_DECODE_STORE_LAG;
constexpr uint32_t kTileBytes = 64 * 128 * 4;  // half of a head's state
constexpr int kComputeThreads = 256;
constexpr int kThreads = kComputeThreads + 32;  // + producer warp
constexpr uint32_t OFF_MISC = kStages * kTileBytes;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4096 + 1024;
}  // namespace dec

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// 16 values per lane -> lane l holds the warp-wide sum of value (l >> 1).
__device__ __forceinline__ float warp_transpose_sum16(float (&v)[16], int lane) {
#pragma unroll
    for (int off = 16, n = 8; off >= 2; off >>= 1, n >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float send = upper ? v[i] : v[i + n];
            const float keep = upper ? v[i + n] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, bool& broken) {
    if (broken) return false;
    if (!mbar_wait(bar, parity)) {
        broken = true;
        record_error(kErrTimeoutTma);
        return false;
    }
    return true;
}

__global__ void __launch_bounds__(dec::kThreads, 1) gdn_decode_kernel(const DecodeParams p) {
    using namespace dec;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_MISC);
    uint64_t* empty = full + kStages;
    float* s_q = reinterpret_cast<float*>(smem + OFF_MISC + 128);
    float* s_k = s_q + 128;
    float* s_v = s_k + 128;
    float* s_o = s_v + 128;
    float* s_red = s_o + 128;     // [16]
    float* s_gate = s_red + 16;   // [4]

    const int h = blockIdx.x;
    const int part = blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int group = p.Vh / p.Kh;
    const int kap = h / group;
    const int nrows = (p.rows > part) ? (p.rows - part + p.P - 1) / p.P : 0;
    const int nunits = 2 * nrows;
    bool broken = false;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kComputeThreads / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();

    auto tile_src = [&](int u) -> float* {
        const int row = part + (u >> 1) * p.P;
        return p.state + (((size_t)row * p.Vh + h) * 128 + (u & 1) * 64) * 128;
    };

    if (warp == kComputeThreads / 32) {
        // ---------------- producer warp
        if (lane == 0) {
            for (int u = 0; u < nunits && u < kStages; ++u) {
                mbar_arrive_expect_tx(&full[u], kTileBytes);
                bulk_load(smem + u * kTileBytes, tile_src(u), kTileBytes, &full[u]);
            }
        }
        for (int j = 0; j < nrows; ++j) {
            cluster_arrive();
            if (lane == 0) {
                for (int half = 0; half < 2; ++half) {
                    const int u = 2 * j + half;
                    const int st = u % kStages;
                    bounded_wait(&empty[st], (u / kStages) & 1, broken);
                    bulk_store(tile_src(u), smem + st * kTileBytes, kTileBytes);
                    bulk_commit();
                    // refill the stage of unit v = u - kStoreLag once its store has read the stage
                    const int v = u - kStoreLag;
                    if (v >= 0 && v + kStages < nunits) {
                        if (kStoreLag == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                        else asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(kStoreLag) : "memory");
                        const int sv = v % kStages;
                        mbar_arrive_expect_tx(&full[sv], kTileBytes);
                        bulk_load(smem + sv * kTileBytes, tile_src(v + kStages), kTileBytes, &full[sv]);
                    }
                }
            }
            __syncwarp();
            cluster_wait();
        }
        if (lane == 0) bulk_wait_all();
        return;
    }

    // ---------------- compute warps (tid < 256)
    // channel slots of this thread: idx = tid (q for tid < 128, k otherwise) and tid + 256 (v, tid < 128)
    int ch[2];
    float w[2][4];
    const int nslots = (tid < 128) ? 2 : 1;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int idx = tid + u * 256;
        const int grp = idx >> 7, c = idx & 127;
        ch[u] = (grp == 0) ? kap * 128 + c : (grp == 1) ? p.Kh * 128 + kap * 128 + c : 2 * p.Kh * 128 + h * 128 + c;
        if (u < nslots) {
            const uint2 wb = *reinterpret_cast<const uint2*>(p.conv_w + (size_t)ch[u] * 4);
            w[u][0] = __uint_as_float(wb.x << 16);
            w[u][1] = __uint_as_float(wb.x & 0xffff0000u);
            w[u][2] = __uint_as_float(wb.y << 16);
            w[u][3] = __uint_as_float(wb.y & 0xffff0000u);
        }
    }
    const bool hist_writer_qk = (h % group) == 0;
    const float A_exp = expf(p.A_log[h]);
    const float dtb = p.dt_bias[h];
    const float wn = (tid < 128) ? 1.0f + p.norm_w[tid] : 0.f;

    // prefetched inputs of the next row (plain registers: h0/h1/h2/x of the two slots, z, a, b)
    float h00 = 0.f, h01 = 0.f, h02 = 0.f, x0 = 0.f, h10 = 0.f, h11 = 0.f, h12 = 0.f, x1 = 0.f;
    float zn = 0.f, an = 0.f, bn = 0.f;
#define GDN_DECODE_PREFETCH(jj)                                                              \
    {                                                                                        \
        const int prow = part + (jj) * p.P;                                                  \
        const float* hr0 = p.conv + (size_t)prow * 3 * p.C + ch[0];                          \
        h00 = hr0[0];                                                                        \
        h01 = hr0[p.C];                                                                      \
        h02 = hr0[2 * p.C];                                                                  \
        x0 = bf16_bits_to_float(p.qkv[(size_t)prow * p.C + ch[0]]);                          \
        if (nslots > 1) {                                                                    \
            const float* hr1 = p.conv + (size_t)prow * 3 * p.C + ch[1];                      \
            h10 = hr1[0];                                                                    \
            h11 = hr1[p.C];                                                                  \
            h12 = hr1[2 * p.C];                                                              \
            x1 = bf16_bits_to_float(p.qkv[(size_t)prow * p.C + ch[1]]);                      \
            zn = bf16_bits_to_float(p.z[(size_t)prow * p.Vh * 128 + h * 128 + tid]);         \
        }                                                                                    \
        if (tid == 0) {                                                                      \
            an = bf16_bits_to_float(p.a[(size_t)prow * p.Vh + h]);                           \
            bn = bf16_bits_to_float(p.b[(size_t)prow * p.Vh + h]);                           \
        }                                                                                    \
    }
    if (nrows > 0) GDN_DECODE_PREFETCH(0);

    for (int j = 0; j < nrows; ++j) {
        const int row = part + j * p.P;
        named_barrier_sync(1, kComputeThreads);  // previous row's readers of s_* are done
        // ---- conv + silu of this row's channels (history was prefetched)
        const float act0 = silu_f(w[0][0] * h00 + w[0][1] * h01 + w[0][2] * h02 + w[0][3] * x0);
        const float act1 = silu_f(w[1][0] * h10 + w[1][1] * h11 + w[1][2] * h12 + w[1][3] * x1);
        const float k00 = h01, k01 = h02, k02 = x0, k10 = h11, k11 = h12, k12 = x1;  // shifted history
        const float zval = zn;
        if (tid == 0) {
            s_gate[0] = -A_exp * softplus_f(an + dtb);
            s_gate[1] = sigmoid_f(bn);
        }
        cluster_arrive();  // this CTA has read the row's history
        if (j + 1 < nrows) GDN_DECODE_PREFETCH(j + 1);

        // ---- L2 norms: q in warps 0-3, k in warps 4-7
        {
            const float ss = warp_sum(act0 * act0);
            if (lane == 0) s_red[warp] = ss;
        }
        named_barrier_sync(1, kComputeThreads);
        {
            const float qss = s_red[0] + s_red[1] + s_red[2] + s_red[3];
            const float kss = s_red[4] + s_red[5] + s_red[6] + s_red[7];
            if (tid < 128) {
                s_q[tid] = act0 * rsqrtf(qss + kEps) * rsqrtf(128.0f);
                s_v[tid] = act1;
            } else {
                s_k[tid - 128] = act0 * rsqrtf(kss + kEps);
            }
        }
        named_barrier_sync(1, kComputeThreads);
        const float4 qf = reinterpret_cast<const float4*>(s_q)[lane];
        const float4 kf = reinterpret_cast<const float4*>(s_k)[lane];
        const float kq = warp_sum(kf.x * qf.x + kf.y * qf.y + kf.z * qf.z + kf.w * qf.w);
        const float alpha = expf(s_gate[0]);
        const float beta = s_gate[1];

        // ---- stream the two half-tiles of the state
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const int u = 2 * j + half;
            const int st = u % kStages;
            bounded_wait(&full[st], (u / kStages) & 1, broken);
            float* tile = reinterpret_cast<float*>(smem + st * kTileBytes);
            float4 s[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) s[r] = reinterpret_cast<const float4*>(tile + (warp * 8 + r) * 128)[lane];
            float vals[16];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                vals[2 * r] = s[r].x * kf.x + s[r].y * kf.y + s[r].z * kf.z + s[r].w * kf.w;
                vals[2 * r + 1] = s[r].x * qf.x + s[r].y * qf.y + s[r].z * qf.z + s[r].w * qf.w;
            }
            const float tot = warp_transpose_sum16(vals, lane);  // lane l: row l>>2, S.k if bit 1 clear else S.q
            const int rr = lane >> 2;
            const int irow = half * 64 + warp * 8 + rr;
            const float u_k = beta * (s_v[irow] - alpha * tot);      // meaningful on lanes 4r, 4r+1
            const float u_r = __shfl_sync(0xffffffffu, u_k, lane & ~3);
            if ((lane & 3) == 2) s_o[irow] = alpha * tot + u_r * kq;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float ur = __shfl_sync(0xffffffffu, u_k, 4 * r);
                float4 n;
                n.x = alpha * s[r].x + ur * kf.x;
                n.y = alpha * s[r].y + ur * kf.y;
                n.z = alpha * s[r].z + ur * kf.z;
                n.w = alpha * s[r].w + ur * kf.w;
                reinterpret_cast<float4*>(tile + (warp * 8 + r) * 128)[lane] = n;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }

        // ---- gated RMSNorm over the head's 128 outputs
        named_barrier_sync(1, kComputeThreads);
        {
            const float o = (tid < 128) ? s_o[tid] : 0.f;
            const float ss = warp_sum(o * o);
            if (lane == 0) s_red[8 + warp] = ss;
        }
        named_barrier_sync(1, kComputeThreads);
        if (tid < 128) {
            const float ms = (s_red[8] + s_red[9] + s_red[10] + s_red[11]) * (1.0f / 128.0f);
            const float y = s_o[tid] * rsqrtf(ms + kEps) * wn * silu_f(zval);
            p.out[(size_t)row * p.Vh * 128 + h * 128 + tid] = float_to_bf16_bits(y);
        }

        // ---- history shift, after every CTA of the cluster has read the old values
        cluster_wait();
        if (hist_writer_qk) {  // slot 0: a q/k channel shared by the cluster
            float* hr = p.conv + (size_t)row * 3 * p.C + ch[0];
            hr[0] = k00;
            hr[p.C] = k01;
            hr[2 * p.C] = k02;
        }
        if (nslots > 1) {  // slot 1: a v channel of this head
            float* hr = p.conv + (size_t)row * 3 * p.C + ch[1];
            hr[0] = k10;
            hr[p.C] = k11;
            hr[2 * p.C] = k12;
        }
    }
}

#undef GDN_DECODE_PREFETCH

}  // namespace gdn
