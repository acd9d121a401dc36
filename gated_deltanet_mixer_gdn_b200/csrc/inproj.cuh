// The load stage fused into the in_proj GEMM's epilogue (prefill from the
// layer's hidden states).  Per token the in_proj product [qkv | z | b | a]
// (module tree of the Qwen3.8 27B architecture page, `linear_attn`) is
// rounded to bf16, exactly as gdn_in_proj writes it, and then goes through
// the same arithmetic, in the same order, as the load stage of prep.cuh
// (Qwen3.8 27B model card, "Gated DeltaNet" bullet): the depthwise causal
// conv (width 4) + silu, the L2 norms of q and k (q also scaled by
// 1/sqrt(128)) with their f16 hi/lo split, the f16 copy of v, the gates of the
// value heads; z is stored as bf16.  The pre-conv values never reach HBM.
//
// An epilogue thread owns one token row of the 128 x 256 tile.  A tile's 128
// rows start 3 tokens before its first output token, so the conv window of
// every output row lies inside the tile: 32 columns at a time, the rows go
// through a shared-memory buffer from which each thread reads the three rows
// before its own; at a row's first tokens the window takes the row's history
// instead.  The L2 norm of a head (128 channels in one thread) is summed in
// the order of the warp reduction of prep.cuh (32 partial sums of 4 channels,
// then the butterfly), so the two paths agree bit for bit.
#pragma once

#include "gemm.cuh"
#include "prep.cuh"

namespace gdn {

__device__ __forceinline__ float bf16_round(float x) { return bf16_bits_to_float(float_to_bf16_bits(x)); }

template <int FUSED>
__device__ void fused_prep_epilogue(const FusedPrep& f, const GemmParams& p, uint32_t tacc, int r0, int n0,
                                    uint8_t* scratch, int q4, int lane) {
    const int C = (2 * f.Kh + f.Vh) * kD;
    const int VD = f.Vh * kD;
    const int lrow = 32 * q4 + lane;  // row of the tile
    const int r = r0 + lrow;          // token (rows before 0 or past M are padding)
    const bool out_row = lrow >= 3 && r < p.M;
    int n = 0, pos = 0, len = f.T;           // packed row of the token, position in it, its length
    if (out_row) {
        if (f.cu == nullptr) {
            n = r / f.T;
            pos = r - n * f.T;
        } else {  // the last row starting at or before r (empty rows share their start with the next)
            int lo = 0, hi = f.N;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(f.cu + mid) <= r) lo = mid;
                else hi = mid;
            }
            n = lo;
            const int start = __ldg(f.cu + n);
            pos = r - start;
            len = __ldg(f.cu + n + 1) - start;
        }
    }
    float* xbuf = reinterpret_cast<float*>(scratch);                          // [128][kXStride]
    float4* taps = reinterpret_cast<float4*>(scratch + gemm::XBUF_BYTES);       // [256] {w0, w1, w2, w3}

    if (n0 < C) {
        // ---------------- q, k or v channels: conv + silu (+ norm and hi/lo for q, k)
        named_barrier_sync(4, 128);  // the previous tile's readers of the taps are done
        {
            const uint4 tw = __ldg(reinterpret_cast<const uint4*>(f.conv_w + (size_t)n0 * 4) + lrow);  // 2 channels
            taps[2 * lrow] = make_float4(__uint_as_float(tw.x << 16), __uint_as_float(tw.x & 0xffff0000u),
                                         __uint_as_float(tw.y << 16), __uint_as_float(tw.y & 0xffff0000u));
            taps[2 * lrow + 1] = make_float4(__uint_as_float(tw.z << 16), __uint_as_float(tw.z & 0xffff0000u),
                                             __uint_as_float(tw.w << 16), __uint_as_float(tw.w & 0xffff0000u));
        }
        const int slot = n0 / kD;  // head slot of the tile's first head: q 0..Kh-1, k Kh..2Kh-1, v after
        const bool is_v = slot >= 2 * f.Kh;
        const bool is_q = slot < f.Kh;
        const bool at_end = out_row && pos >= len - 3;  // one of the row's last three tokens
        const int rm[3] = {max(lrow - 1, 0), max(lrow - 2, 0), max(lrow - 3, 0)};  // rows 0-2 only pad
        // conv + silu of channels [32 j, 32 j + 32) of head hh of the tile
        auto conv_chunk = [&](int hh, int j, float* act) {
            const int cb = 128 * hh + 32 * j;  // first column of the chunk in the tile
            float v[32];
            tmem_ld32(tacc + cb, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const uint32_t pk = pack_bf16x2(v[e], v[e + 1]);  // the projection as bf16
                v[e] = __uint_as_float(pk << 16);
                v[e + 1] = __uint_as_float(pk & 0xffff0000u);
            }
            named_barrier_sync(4, 128);  // the buffer's previous readers (and the taps' writers) are done
            float4* xr = reinterpret_cast<float4*>(xbuf + lrow * gemm::kXStride);
#pragma unroll
            for (int q = 0; q < 8; ++q) xr[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            if (at_end) {
                float4* dst = reinterpret_cast<float4*>(f.conv_last + ((size_t)n * 3 + pos + 3 - len) * C + n0 + cb);
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = xr[q];
            }
            named_barrier_sync(4, 128);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float4 x1 = reinterpret_cast<const float4*>(xbuf + rm[0] * gemm::kXStride)[q];  // x[t-1]
                float4 x2 = reinterpret_cast<const float4*>(xbuf + rm[1] * gemm::kXStride)[q];  // x[t-2]
                float4 x3 = reinterpret_cast<const float4*>(xbuf + rm[2] * gemm::kXStride)[q];  // x[t-3]
                if (out_row && pos < 3) {  // the row's history (or zeros) before its first token
                    const float* h = f.init_conv ? f.init_conv + (size_t)n * 3 * C + n0 + cb + 4 * q : nullptr;
                    auto hist = [&](int xi) {  // index xi of the history [3][C]
                        return h ? *reinterpret_cast<const float4*>(h + (size_t)xi * C) : make_float4(0.f, 0.f, 0.f, 0.f);
                    };
                    if (pos < 1) x1 = hist(2 + pos);
                    if (pos < 2) x2 = hist(1 + pos);
                    x3 = hist(pos);
                }
                const float xa[4] = {x1.x, x1.y, x1.z, x1.w}, xb[4] = {x2.x, x2.y, x2.z, x2.w};
                const float xc[4] = {x3.x, x3.y, x3.z, x3.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 t = taps[cb + 4 * q + e];
                    act[4 * q + e] = silu_f(fmaf(t.x, xc[e], fmaf(t.y, xb[e], fmaf(t.z, xa[e], t.w * v[4 * q + e]))));
                }
            }
        };
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
            const int hslot = slot + hh;
            if (is_v) {
#pragma unroll 1
                for (int j = 0; j < 4; ++j) {
                    float act[32];
                    conv_chunk(hh, j, act);
                    if (out_row) {
                        uint4* dst = reinterpret_cast<uint4*>(f.Vs + (size_t)r * VD + (hslot - 2 * f.Kh) * kD + 32 * j);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 pk;
                            pk.x = pack_half2(act[8 * q + 0], act[8 * q + 1]);
                            pk.y = pack_half2(act[8 * q + 2], act[8 * q + 3]);
                            pk.z = pack_half2(act[8 * q + 4], act[8 * q + 5]);
                            pk.w = pack_half2(act[8 * q + 6], act[8 * q + 7]);
                            dst[q] = pk;
                        }
                    }
                }
                continue;
            }
            // q / k: the whole head in registers, then the squared norm in the order of
            // prep.cuh (32 partial sums of 4 channels, then the xor butterfly)
            float act[128];
#pragma unroll
            for (int j = 0; j < 4; ++j) conv_chunk(hh, j, act + 32 * j);
            float part[32];
#pragma unroll
            for (int l = 0; l < 32; ++l) {
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) ss = fmaf(act[4 * l + e], act[4 * l + e], ss);
                part[l] = ss;
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
                for (int l = 0; l < o; ++l) part[l] = part[l] + part[l + o];
            float scale = rsqrtf(part[0] + kEps);
            if (is_q) scale *= rsqrtf((float)kD);
            if (out_row) {
                const size_t off = (size_t)r * f.Kh * kD + (is_q ? hslot : hslot - f.Kh) * kD;
                uint4* dh = reinterpret_cast<uint4*>((is_q ? f.Qs : f.Ks) + off);
                uint4* dl = reinterpret_cast<uint4*>((is_q ? f.Ql : f.Kl) + off);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float xa = __fmul_rn(act[8 * q + 2 * e], scale);
                        const float xb = __fmul_rn(act[8 * q + 2 * e + 1], scale);
                        hw[e] = pack_half2(xa, xb);
                        const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hw[e]));
                        lw[e] = pack_half2(xa - hf.x, xb - hf.y);
                    }
                    dh[q] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    dl[q] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
        }
    } else if (n0 < C + VD) {
        // ---------------- z: bf16
#pragma unroll 1
        for (int j = 0; j < gemm::BN / 32; ++j) {
            float v[32];
            tmem_ld32(tacc + 32 * j, v);
            tmem_ld_wait();
            if (out_row) {
                uint4* dst = reinterpret_cast<uint4*>(f.z + (size_t)r * VD + (n0 - C) + 32 * j);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    uint4 pk;
                    pk.x = pack_bf16x2(v[8 * e + 0], v[8 * e + 1]);
                    pk.y = pack_bf16x2(v[8 * e + 2], v[8 * e + 3]);
                    pk.z = pack_bf16x2(v[8 * e + 4], v[8 * e + 5]);
                    pk.w = pack_bf16x2(v[8 * e + 6], v[8 * e + 7]);
                    dst[e] = pk;
                }
            }
        }
    } else {
        // ---------------- b, a (Vh each): the gates of the value heads
#pragma unroll 1
        for (int j = 0; j < (2 * f.Vh + 31) / 32; ++j) {  // b in columns 0..Vh-1, a in Vh..2Vh-1
            float v[32];
            tmem_ld32(tacc + 32 * j, v);
            tmem_ld_wait();
            if (out_row) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int c = 32 * j + e;
                    if (c < f.Vh) {
                        f.Bs[(size_t)c * p.M + r] = sigmoid_f(bf16_round(v[e]));
                    } else if (c < 2 * f.Vh) {
                        const int h = c - f.Vh;
                        f.Gs[(size_t)h * p.M + r] =
                            -expf(__ldg(f.A_log + h)) * softplus_f(bf16_round(v[e]) + __ldg(f.dt_bias + h));
                    }
                }
            }
        }
    }
}

// Final histories after the fused load stage: row n's history after its len tokens is rows
// len .. len + 2 of [initial history (3 rows); the row's tokens].  The epilogue staged the
// row's last min(len, 3) pre-conv tokens (token pos in slot pos + 3 - len); the other rows
// come from the initial history (zeros without one).  final_conv may alias init_conv: for each
// channel the thread reads initial row j + len before writing row j, in increasing j.
__global__ void __launch_bounds__(256) gdn_conv_merge_kernel(SeqIndex seq, int C, const float* staged,
                                                             const float* init_conv, float* final_conv) {
    const int n = blockIdx.y;
    const int ch = blockIdx.x * blockDim.x + threadIdx.x;
    if (ch >= C) return;
    int start, len;
    seq.bounds(n, start, len);
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        float v;
        if (j >= 3 - len) v = staged[((size_t)n * 3 + j) * C + ch];
        else v = init_conv ? init_conv[((size_t)n * 3 + j + len) * C + ch] : 0.f;
        final_conv[((size_t)n * 3 + j) * C + ch] = v;
    }
}

}  // namespace gdn
