// Load stage of the chunked prefill: per token, the depthwise causal conv
// (width 4) + silu over all qkv channels, L2 normalisation of the q and k
// heads (q also scaled by 1/sqrt(128)), and the two gates of every value head
// (Qwen3.8 27B model card, "Gated DeltaNet" bullet).  Results are staged as
// f16 operands for the tensor-core chunk kernel:
//   Qs, Ks  f16 [total][Kh*128]   (q / (|q| sqrt(128)), k / |k|)
//   Vs      f16 [total][Vh*128]
//   Gs, Bs  f32 [Vh][total]       (g = log-decay, beta = write rate)
// A second tiny kernel writes each row's final conv history.
//
// Mapping: a warp owns one 128-channel head slot, each lane 4 contiguous
// channels (8-byte loads and stores), so the per-token L2 norm is one warp
// shuffle reduction.
#pragma once

#include "common.cuh"

namespace gdn {

struct SeqIndex {
    const int* cu;   // device cu_seqlens [N+1], or nullptr for uniform rows
    int uniform_T;   // row length when cu == nullptr
    int N;
    __device__ __forceinline__ void locate(int t, int& n, int& start, int& len) const {
        if (cu == nullptr) {
            n = t / uniform_T;
            start = n * uniform_T;
            len = uniform_T;
            return;
        }
        int lo = 0, hi = N;  // find n with cu[n] <= t < cu[n+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(cu + mid) <= t) lo = mid;
            else hi = mid;
        }
        // skip empty rows that share the same start
        n = lo;
        start = __ldg(cu + n);
        len = __ldg(cu + n + 1) - start;
    }
    __device__ __forceinline__ void bounds(int n, int& start, int& len) const {
        if (cu == nullptr) {
            start = n * uniform_T;
            len = uniform_T;
        } else {
            start = __ldg(cu + n);
            len = __ldg(cu + n + 1) - start;
        }
    }
};

struct PrepParams {
    int Kh, Vh, C, total;
    int tok_begin, tok_end;   // tokens processed by this launch
    SeqIndex seq;
    const uint16_t* qkv;      // bf16 [total][C]
    const uint16_t* a;        // bf16 [total][Vh]
    const uint16_t* b;        // bf16 [total][Vh]
    const uint16_t* conv_w;   // bf16 [C][4]
    const float* A_log;
    const float* dt_bias;
    const float* init_conv;   // f32 [N or pool][3][C] or nullptr
    const int* slots;         // [N] history row of each packed row (validated by the host), or nullptr
    __half* Qs;
    __half* Ks;
    __half* Ql;
    __half* Kl;
    __half* Vs;
    float* Gs;
    float* Bs;
};

template <bool B>
struct Flag {
    static constexpr bool value = B;
};

constexpr int kPrepTokens = 16;  // consecutive tokens per thread
constexpr int kPrepSlots = 8;    // head slots (warps) per CTA
// The CTA's input rows (3 before its first token, for the conv window, then its tokens) x its
// 1024 channels, staged in shared memory by TMA at the start: 4 boxes of 256 channels.
constexpr int kPrepRows = kPrepTokens + 3;
constexpr int kPrepBox = 256;
constexpr uint32_t kPrepBlockBytes = kPrepRows * kPrepBox * 2;               // 9,728
constexpr uint32_t kPrepTileBytes = (kPrepSlots * kD / kPrepBox) * kPrepBlockBytes;  // 38,912
constexpr uint32_t kPrepSmem = kPrepTileBytes + 16 + 128;                   // + barrier, alignment

__device__ __forceinline__ void unpack4(const uint2 v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xffff0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xffff0000u);
}

// A CTA covers 8 head slots (one warp each, 4 channels per lane) for
// kPrepTokens consecutive tokens.  Its input rows arrive in shared memory by TMA
// all at once (about 38 KB in flight per CTA, rows outside the tensor read as
// zero); each thread keeps its taps unpacked and the last three inputs of its
// channels in registers (a rolling window that restarts from the row's history
// at every row start): per token one 8-byte shared-memory read and a short
// instruction chain per thread, with many warps resident per SM.
__global__ void __launch_bounds__(256, 4) gdn_prep_kernel(const __grid_constant__ CUtensorMap tmX, const PrepParams p) {
    const int lane = threadIdx.x & 31;
    const int nheads = 2 * p.Kh + p.Vh;
    const int wslot = threadIdx.x >> 5;
    const int slot = blockIdx.y * kPrepSlots + wslot;
    const int t0 = p.tok_begin + blockIdx.x * kPrepTokens;
    const int nt = min(kPrepTokens, p.tok_end - t0);
    if (nt <= 0) return;  // whole CTA

    extern __shared__ uint8_t prep_smem_raw[];
    uint8_t* tile = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(prep_smem_raw) + 127) & ~uintptr_t(127));
    uint64_t* bar = reinterpret_cast<uint64_t*>(tile + kPrepTileBytes);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(bar, kPrepTileBytes);
#pragma unroll
        for (int i = 0; i < (int)(kPrepSlots * kD / kPrepBox); ++i)
            tma_load_2d(tile + i * kPrepBlockBytes, &tmX, blockIdx.y * kPrepSlots * kD + i * kPrepBox, t0 - 3, bar);
    }
    __syncthreads();  // the barrier is initialised before anyone waits on it
    if (slot >= nheads) return;  // whole warp
    const int ch0 = slot * kD + lane * 4;
    const bool is_q = slot < p.Kh;
    const bool is_v = slot >= 2 * p.Kh;
    const int vh = slot - 2 * p.Kh;
    // this lane's 4 channels in input row r of the tile (r = token - t0 + 3)
    const uint8_t* xcol = tile + (wslot >> 1) * kPrepBlockBytes + ((wslot & 1) * kD + lane * 4) * 2;
    auto xrow = [&](int r) { return *reinterpret_cast<const uint2*>(xcol + r * kPrepBox * 2); };
    float w[4][4];  // w[j][e]: tap j of channel ch0 + e
    {
        const uint4* wp = reinterpret_cast<const uint4*>(p.conv_w + (size_t)ch0 * 4);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 v = __ldg(wp + q);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int e = q * 2 + m / 2;  // two channels per uint4 (8 bf16 = 2 x 4 taps)
                const int j = (m % 2) * 2;
                w[j][e] = __uint_as_float(u[m] << 16);
                w[j + 1][e] = __uint_as_float(u[m] & 0xffff0000u);
            }
        }
    }
    if (is_v && lane < nt && GDN_CHECK(t0 + lane < p.total && vh < p.Vh)) {  // gates: one token per lane
        const int t = t0 + lane;
        const float av = bf16_bits_to_float(p.a[(size_t)t * p.Vh + vh]);
        const float bv = bf16_bits_to_float(p.b[(size_t)t * p.Vh + vh]);
        p.Gs[(size_t)vh * p.total + t] = -expf(__ldg(p.A_log + vh)) * softplus_f(av + __ldg(p.dt_bias + vh));
        p.Bs[(size_t)vh * p.total + t] = sigmoid_f(bv);
    }

    if (!mbar_wait(bar, 0)) {  // the tile never landed: recorded, nothing written
        record_error(kErrTimeoutTma);
        return;
    }
    int n, start, len;
    p.seq.locate(t0, n, start, len);
    // window: w0 = index s, w1 = s + 1, w2 = s + 2 of [history (3 rows); tokens of the row]
    float w0[4], w1[4], w2[4];
    auto fetch_xbar = [&](int nn, int xi, int tok, float (&x)[4]) {
        if (xi >= 3) {  // a token of the row: one of the tile's three rows before t0
            if (GDN_CHECK(tok >= t0 - 3 && tok < t0 && tok >= 0 && ch0 + 4 <= p.C)) unpack4(xrow(tok - t0 + 3), x);
        } else if (p.init_conv != nullptr && GDN_CHECK(nn >= 0 && nn < p.seq.N && xi >= 0)) {
            const int sr = p.slots ? __ldg(p.slots + nn) : nn;
            const float4 h = __ldg(reinterpret_cast<const float4*>(p.init_conv + ((size_t)sr * 3 + xi) * p.C + ch0));
            x[0] = h.x; x[1] = h.y; x[2] = h.z; x[3] = h.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = 0.f;
        }
    };
    {
        const int s = t0 - start;
        fetch_xbar(n, s, t0 - 3, w0);
        fetch_xbar(n, s + 1, t0 - 2, w1);
        fetch_xbar(n, s + 2, t0 - 1, w2);
    }

    // The token loop, instantiated for v / q-k slots and for blocks that lie inside one row
    // (FAST: no row start to watch for, no ragged end, so the 16 tokens are straight-line
    // code the compiler can interleave) or not.
    auto run = [&](auto v_flag, auto fast_flag) {
        constexpr bool IS_V = decltype(v_flag)::value;
        constexpr bool FAST = decltype(fast_flag)::value;
#pragma unroll
        for (int tt = 0; tt < kPrepTokens; ++tt) {
            if (!FAST && tt >= nt) break;
            const int t = t0 + tt;
            if (!GDN_CHECK(t < p.total)) break;
            float xn[4];
            unpack4(xrow(tt + 3), xn);
            if (!FAST && t == start + len) {  // a new row starts here (skip empty rows): restart from its history
                if (p.seq.cu == nullptr) {
                    ++n;
                    start += len;
                } else {
                    do {
                        ++n;
                        start = __ldg(p.seq.cu + n);
                        len = __ldg(p.seq.cu + n + 1) - start;
                    } while (len == 0);
                }
                fetch_xbar(n, 0, 0, w0);
                fetch_xbar(n, 1, 0, w1);
                fetch_xbar(n, 2, 0, w2);
            }
            float act[4];
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float cv = fmaf(w[0][e], w0[e], fmaf(w[1][e], w1[e], fmaf(w[2][e], w2[e], w[3][e] * xn[e])));
                act[e] = silu_f(cv);
                ss = fmaf(act[e], act[e], ss);
                w0[e] = w1[e];
                w1[e] = w2[e];
                w2[e] = xn[e];
            }
            float scale = 1.0f;
            if constexpr (!IS_V) {
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                scale = rsqrtf(ss + kEps);
                if (is_q) scale *= rsqrtf((float)kD);
            }
            float xs[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) xs[e] = __fmul_rn(act[e], scale);  // rounded product (no contraction into the lo split)
            uint2 pk;
            pk.x = pack_half2(xs[0], xs[1]);
            pk.y = pack_half2(xs[2], xs[3]);
            if constexpr (IS_V) {
                *reinterpret_cast<uint2*>(p.Vs + (size_t)t * p.Vh * kD + vh * kD + lane * 4) = pk;
            } else {
                const size_t off = (size_t)t * p.Kh * kD + (is_q ? slot : slot - p.Kh) * kD + lane * 4;
                const float2 h0 = __half22float2(*reinterpret_cast<const __half2*>(&pk.x));
                const float2 h1 = __half22float2(*reinterpret_cast<const __half2*>(&pk.y));
                uint2 lo;
                lo.x = pack_half2(xs[0] - h0.x, xs[1] - h0.y);
                lo.y = pack_half2(xs[2] - h1.x, xs[3] - h1.y);
                *reinterpret_cast<uint2*>((is_q ? p.Qs : p.Ks) + off) = pk;
                *reinterpret_cast<uint2*>((is_q ? p.Ql : p.Kl) + off) = lo;
            }
        }
    };
    const bool fast = nt == kPrepTokens && t0 + kPrepTokens <= start + len;  // CTA-uniform
    if (is_v) {
        if (fast) run(Flag<true>{}, Flag<true>{});
        else run(Flag<true>{}, Flag<false>{});
    } else {
        if (fast) run(Flag<false>{}, Flag<true>{});
        else run(Flag<false>{}, Flag<false>{});
    }
}


struct ConvOutParams {
    int C, N, total;
    SeqIndex seq;
    const uint16_t* qkv;     // bf16 [total][C]
    const float* init_conv;  // f32 [N or pool][3][C] or nullptr
    float* final_conv;       // f32 [N or pool][3][C]; may alias init_conv
    const int* slots;        // [N] history row of each packed row, or nullptr
};

// final_conv[n][r] = row L+r of [history (3 rows); the row's L tokens].
// In place is safe: for each channel the thread reads index L+r >= r before
// writing index r, in increasing r.
__global__ void __launch_bounds__(256) gdn_conv_out_kernel(const ConvOutParams p) {
    const int n = blockIdx.y;
    const int ch = blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= p.C) return;
    int start, len;
    p.seq.bounds(n, start, len);
    if (!GDN_CHECK(n < p.N && start >= 0 && len >= 0)) return;
    const size_t sr = p.slots ? (size_t)__ldg(p.slots + n) : (size_t)n;
#pragma unroll
    for (int r = 0; r < 3; ++r) {
        const int e = len + r;
        float v;
        if (e >= 3) v = GDN_CHECK(start + e - 3 < p.total) ? bf16_bits_to_float(p.qkv[(size_t)(start + e - 3) * p.C + ch]) : 0.f;
        else v = p.init_conv ? p.init_conv[(sr * 3 + e) * p.C + ch] : 0.f;
        p.final_conv[(sr * 3 + r) * p.C + ch] = v;
    }
}

}  // namespace gdn
