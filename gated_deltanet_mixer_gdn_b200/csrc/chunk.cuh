// Chunked prefill of the gated delta rule on 5th-generation tensor cores:
// the state recurrence over the chunks of a row, and the gated-RMSNorm output.
//
// The recurrence (Qwen3.8 27B model card, "Gated DeltaNet" bullet), per value
// head with state S [128 v][128 k]:
//     S_t = exp(g_t) S_{t-1} + u_t k_t^T,   u_t = beta_t (v_t - exp(g_t) S_{t-1} k_t),
//     o_t = S_t q_t.
// Over a chunk of 64 tokens, with the per-chunk record of wy.cuh (T1, W, M
// and the decays, none of which depends on the state):
//     U   = T1 V - W S0^T                                   (U~ = T1 V)
//     O   = diag(e^G) Q S0^T + M U
//     S_C = e^{G_C} S0 + U^T diag(e^{G_C - G}) K.
//
// One CTA owns one (row, value head) and walks its chunks in order.  Two
// warp-specialised groups run side by side:
//   * the chain (8 warps) carries the state: MMA4 U^T = U~^T - S0 W^T and
//     MMA5 Oi^T = S0 Q^T with S0 as f16 in shared memory; U^T to f16 in TMEM
//     (plain, and scaled by e^{G_C - G}); MMA6 S += (U^T diag e^{G_C-G}) K and
//     MMA7 Oa^T = U^T M^T with A read from TMEM; then the f16 copy of the new
//     state and its scaling by the next chunk's e^{G_C}.  Its thread 0 also
//     issues the loads of chunk c+2 and MMA2 U~^T = V^T T1^T of chunk c+1;
//   * the epilogue (8 warps) turns Oi, Oa of chunk c into o = e^G Oi + Oa,
//     the gated RMSNorm and the bf16 output while the chain is on chunk c+1
//     (double-buffered accumulators).
// Every contraction is a tcgen05.mma with M = 128 and an f32 accumulator in
// TMEM.
#pragma once

#include "common.cuh"
#include "prep.cuh"
#include "wy.cuh"

namespace gdn {

struct ChunkParams {
    int Kh, Vh, total;
    SeqIndex seq;
    const int* chunk_base;    // [N+1] first chunk of each row (varlen), or nullptr for uniform rows
    const uint8_t* rec;       // per-chunk records [nchunks][Vh] (wy.cuh)
    const float* init_state;  // f32 [N][Vh][128][128] or nullptr
    float* final_state;       // f32 [N][Vh][128][128] or nullptr (may alias init_state)
    const float* norm_w;      // f32 [128]
    uint16_t* out;            // bf16 [total][Vh*128]
};

namespace chunk {
constexpr int C = 64;              // tokens per chunk
constexpr int kCThreads = 256;     // state chain, warps 0-7
constexpr int kEThreads = 256;     // epilogue, warps 8-15
constexpr int kThreads = kCThreads + kEThreads;
// one input buffer: K, Q, V f16 [64 t][64] x 2 column blocks (TMA, 128B swizzle), then the record
constexpr uint32_t BUF_K = 0, BUF_Q = 16384, BUF_V = 32768, BUF_REC = 49152;
constexpr uint32_t BUF_BYTES = BUF_REC + 33792;  // record rounded up to 1 KB
// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_BUF0 = 0;
constexpr uint32_t OFF_BUF1 = BUF_BYTES;
constexpr uint32_t OFF_S16 = 2 * BUF_BYTES;      // S0 f16 [128 v][64 k] x 2 blocks
constexpr uint32_t OFF_Z = OFF_S16 + 32768;      // z bf16 [64 t][128], plain row-major; the output tile
constexpr uint32_t OFF_MISC = OFF_Z + 16384;
constexpr uint32_t MISC_BYTES = 3072;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
// misc: 0 barriers, 128 TMEM slot, 256 e^G [4][64] (by chunk mod 4), 1280 reductions [4][64], 2304 rstd[64]
// TMEM columns (f32, 128 lanes)
constexpr uint32_t T_U0 = 0, T_U1 = 64, T_S = 128, T_O0 = 256, T_O1 = 384;  // O: Oi at +0, Oa at +64
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t LD_BYTES = 3 * 16384 + wy::REC_BYTES;
constexpr uint32_t Z_BYTES = 64 * 128 * 2;
constexpr uint32_t ID_KK = idesc_f16_f32(128, 64, false, false, false);
constexpr uint32_t ID_AMN = idesc_f16_f32(128, 64, true, false, false);
constexpr uint32_t ID_NEG_BMN = idesc_f16_f32(128, 64, false, true, true);
constexpr uint32_t ID_DS = idesc_f16_f32(128, 128, false, true, false);
// mbarrier slots
constexpr int B_LD = 0, B_S = 2, B_O = 3, B_E = 5, B_Z = 7;  // B_LD, B_O, B_E: + buffer
constexpr int kBars = 8;
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace chunk

// Lane l of the warp ends with sum over the 32 lanes of v[l] (31 shuffles).
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(chunk::kThreads, 1)
    gdn_chunk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmZ,
                     const __grid_constant__ CUtensorMap tmO, const ChunkParams p) {
    using namespace chunk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);

    const int h = blockIdx.x;
    const int n = blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int kap = h / (p.Vh / p.Kh);
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int hf = (warp >> 2) & 1;           // column half within the group
    const int row = 32 * q4 + lane;           // v row of the state / output channel
    const uint32_t tlane = (static_cast<uint32_t>(32 * q4) << 16);

    uint8_t* misc = smem + OFF_MISC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc + 128);
    float* s_eG = reinterpret_cast<float*>(misc + 256);     // [4][64]
    float* s_red = reinterpret_cast<float*>(misc + 1280);   // [4][64]
    float* s_rstd = reinterpret_cast<float*>(misc + 2304);  // [64]

    int start, len;
    p.seq.bounds(n, start, len);
    const int nchunks = (len + C - 1) / C;
    const int cbase = p.chunk_base ? __ldg(p.chunk_base + n) : n * ((p.seq.uniform_T + C - 1) / C);

    if (tid == 0) {
        mbar_init(&bars[B_LD], 1);
        mbar_init(&bars[B_LD + 1], 1);
        mbar_init(&bars[B_S], 1);
        mbar_init(&bars[B_O], 2);  // the chain's arrive (e^G published) + the commit of MMA7
        mbar_init(&bars[B_O + 1], 2);
        mbar_init(&bars[B_E], 1);
        mbar_init(&bars[B_E + 1], 1);
        mbar_init(&bars[B_Z], 1);
        fence_barrier_init();
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmZ);
        prefetch_tensormap(&tmO);
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *s_tmem;

    auto buf = [&](int c) { return smem + ((c & 1) ? OFF_BUF1 : OFF_BUF0); };
    auto load_chunk = [&](int c) {
        uint8_t* B = buf(c);
        uint64_t* bar = &bars[B_LD + (c & 1)];
        const int y = start + c * C;
        mbar_arrive_expect_tx(bar, LD_BYTES);
        tma_load_2d(B + BUF_K, &tmK, kap * 128, y, bar);
        tma_load_2d(B + BUF_K + 8192, &tmK, kap * 128 + 64, y, bar);
        tma_load_2d(B + BUF_Q, &tmQ, kap * 128, y, bar);
        tma_load_2d(B + BUF_Q + 8192, &tmQ, kap * 128 + 64, y, bar);
        tma_load_2d(B + BUF_V, &tmV, h * 128, y, bar);
        tma_load_2d(B + BUF_V + 8192, &tmV, h * 128 + 64, y, bar);
        bulk_load(B + BUF_REC, p.rec + ((size_t)(cbase + c) * p.Vh + h) * wy::REC_BYTES, wy::REC_BYTES, bar);
    };
    auto load_z = [&](int c) {
        mbar_arrive_expect_tx(&bars[B_Z], Z_BYTES);
        tma_load_2d(smem + OFF_Z, &tmZ, h * 128, start + c * C, &bars[B_Z]);
    };
    // MMA2: U~^T = V^T T1^T of chunk c into its U buffer
    auto mma2 = [&](int c) {
        const uint32_t B = smem_u32(buf(c));
        const uint32_t tU = tbase + ((c & 1) ? T_U1 : T_U0);
#pragma unroll
        for (int s = 0; s < 4; ++s)
            mma_f16(tU, sw128_desc(B + BUF_V + s * 2048, 8192, 1024),
                    sw128_desc(B + BUF_REC + wy::REC_T1 + s * 32, 16, 1024), ID_AMN, s > 0);
    };
    if (tid == 0 && nchunks > 0) {
        load_chunk(0);
        if (nchunks > 1) load_chunk(1);
        load_z(0);
    }
    bool broken = false;
    // every thread of the warp calls this; the warp is converged again on return
    auto wait = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
        __syncwarp();
    };
    // the same for a single thread
    auto wait1 = [&](int slot, uint32_t parity) {
        if (!broken && !mbar_wait(&bars[slot], parity)) {
            broken = true;
            record_error(kErrTimeoutTma);
        }
    };

    if (tid < kCThreads) {
        // =================================================================== state chain
        const int ct = tid;
        // initial state: f16 copy in shared memory, f32 in TMEM scaled by the first chunk's e^{G_C}
        {
            float gC = 1.f;
            if (nchunks > 0) {
                wait(B_LD, 0);
                gC = reinterpret_cast<const float*>(buf(0) + BUF_REC + wy::REC_GATE)[63];
            }
            const float* src =
                p.init_state ? p.init_state + (((size_t)n * p.Vh + h) * 128 + row) * 128 + 64 * hf : nullptr;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 f = src ? __ldg(reinterpret_cast<const float4*>(src + 32 * half) + j)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                    v[4 * j] = f.x;
                    v[4 * j + 1] = f.y;
                    v[4 * j + 2] = f.z;
                    v[4 * j + 3] = f.w;
                }
                store_row_f16_sw128(smem + OFF_S16 + 16384 * hf, row, 4 * half, v, 1.f);
                uint32_t r[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
                tmem_st32(tbase + tlane + T_S + 64 * hf + 32 * half, r);
            }
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_barrier_sync(2, kCThreads);
        if (ct == 0 && nchunks > 0) {
            tc_fence_after();
            mma2(0);
        }
        __syncwarp();

        uint32_t sphase = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const uint32_t aB = smem_u32(buf(c));
            const float* gate = reinterpret_cast<const float*>(buf(c) + BUF_REC + wy::REC_GATE);
            const uint32_t tU = tbase + (b ? T_U1 : T_U0);
            const uint32_t tO = tbase + (b ? T_O1 : T_O0);

            // ---- MMA4: U^T = U~^T - S0 W^T ; MMA5: Oi^T = S0 Q^T
            if (ct == 0) {
                if (c >= 2) wait1(B_E + b, ((c - 2) >> 1) & 1);  // the epilogue is done with O[b]
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t a = sw128_desc(sbase + OFF_S16 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                    mma_f16(tU, a, sw128_desc(aB + BUF_REC + wy::REC_WT + s * 2048, 8192, 1024), ID_NEG_BMN, 1);
                }
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t a = sw128_desc(sbase + OFF_S16 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
                    mma_f16(tO, a, sw128_desc(aB + BUF_Q + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), ID_KK, s > 0);
                }
                mma_commit(&bars[B_S]);
            }
            __syncwarp();
            wait(B_S, sphase);
            sphase ^= 1;
            tc_fence_after();

            // ---- U^T to f16 in TMEM (plain, and scaled by e^{G_C - G_t})
            {
                float u[32];
                tmem_ld32(tU + tlane + 32 * hf, u);
                tmem_ld_wait();
                named_barrier_sync(2, kCThreads);  // every f32 U^T column is read before the f16 copies land
                const float* dec = gate + 64;
                uint32_t uh[16], us[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int t = 32 * hf + 2 * j;
                    uh[j] = pack_half2(u[2 * j], u[2 * j + 1]);
                    us[j] = pack_half2(u[2 * j] * dec[t], u[2 * j + 1] * dec[t + 1]);
                }
                tmem_st16(tU + tlane + 16 * hf, uh);
                tmem_st16(tU + tlane + 32 + 16 * hf, us);
                tmem_st_wait();
                if (ct < 64) s_eG[(c & 3) * 64 + ct] = gate[ct];
            }
            tc_fence_before();
            named_barrier_sync(2, kCThreads);

            // ---- MMA6: S += (U^T diag e^{G_C-G}) K ; MMA7: Oa^T = U^T M^T  (A from TMEM)
            if (ct == 0) {
                mbar_arrive(&bars[B_O + b]);  // e^G of chunk c is published
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(tbase + T_S, tU + 32 + 8 * s, sw128_desc(aB + BUF_K + s * 2048, 8192, 1024), ID_DS, 1);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(tO + 64, tU + 8 * s, sw128_desc(aB + BUF_REC + wy::REC_M + s * 32, 16, 1024), ID_KK,
                               s > 0);
                mma_commit(&bars[B_S]);
                mma_commit(&bars[B_O + b]);
                // the other U buffer is free again: U~ of the next chunk
                if (c + 1 < nchunks) {
                    wait1(B_LD + (b ^ 1), ((c + 1) >> 1) & 1);
                    tc_fence_after();
                    mma2(c + 1);
                }
            }
            __syncwarp();
            wait(B_S, sphase);
            sphase ^= 1;
            tc_fence_after();
            // every input of chunk c has been read: its buffer takes chunk c+2
            if (ct == 0 && c + 2 < nchunks) load_chunk(c + 2);
            __syncwarp();

            // ---- f16 copy of the new state for MMA4/5 of chunk c+1; the f32 state scaled by its e^{G_C}
            if (c + 1 < nchunks) {
                wait(B_LD + (b ^ 1), ((c + 1) >> 1) & 1);
                const float gC = reinterpret_cast<const float*>(buf(c + 1) + BUF_REC + wy::REC_GATE)[63];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tbase + tlane + T_S + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
                    store_row_f16_sw128(smem + OFF_S16 + 16384 * hf, row, 4 * half, v, 1.f);
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
                    tmem_st32(tbase + tlane + T_S + 64 * hf + 32 * half, r);
                }
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                named_barrier_sync(2, kCThreads);
            }
        }

        if (!broken && p.final_state != nullptr) {
            float* dst = p.final_state + (((size_t)n * p.Vh + h) * 128 + row) * 128 + 64 * hf;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tmem_ld32(tbase + tlane + T_S + 64 * hf + 32 * half, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    reinterpret_cast<float4*>(dst + 32 * half)[j] =
                        make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            }
        }
    } else {
        // =================================================================== epilogue
        const int et = tid - kCThreads;
        const float wn = 1.0f + __ldg(p.norm_w + row);  // (1 + w) of this thread's v channel
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int tok0 = start + c * C;
            const int nv = min(C, len - c * C);
            const uint32_t tO = tbase + (b ? T_O1 : T_O0);
            wait(B_O + b, (c >> 1) & 1);
            tc_fence_after();
            float o[32];
            {
                float oa[32];
                tmem_ld32(tO + tlane + 32 * hf, o);
                tmem_ld32(tO + tlane + 64 + 32 * hf, oa);
                tmem_ld_wait();
                tc_fence_before();
                const float* eG = s_eG + (c & 3) * 64 + 32 * hf;
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    o[jj] = fmaf(eG[jj], o[jj], oa[jj]);
                    oa[jj] = o[jj] * o[jj];
                }
                s_red[q4 * 64 + 32 * hf + lane] = warp_transpose_sum(oa, lane);
            }
            named_barrier_sync(3, kEThreads);
            if (et == 0) mbar_arrive(&bars[B_E + b]);  // O[b] may take chunk c+2
            if (et < 64)
                s_rstd[et] = rsqrtf((s_red[et] + s_red[64 + et] + s_red[128 + et] + s_red[192 + et]) * (1.0f / 128.0f) +
                                    kEps);
            named_barrier_sync(3, kEThreads);
            wait(B_Z, c & 1);
            // a full chunk is written over its z tile and leaves by one TMA store; a ragged
            // last chunk is stored directly (the rows past it belong to the next sequence)
            // (the branch stays outside the loops so that their elements can overlap)
            const bool full = (nv == C);
            uint16_t* zt = reinterpret_cast<uint16_t*>(smem + OFF_Z) + 32 * hf * 128 + row;
            const float* rs = s_rstd + 32 * hf;
            if (full) {
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const float zv = bf16_bits_to_float(zt[jj * 128]);
                    zt[jj * 128] = float_to_bf16_bits(o[jj] * rs[jj] * wn * silu_f(zv));
                }
                fence_proxy_async_smem();
            } else {
                uint16_t* op = p.out + (size_t)(tok0 + 32 * hf) * p.Vh * 128 + h * 128 + row;
                const int nt = nv - 32 * hf;  // tokens of this half inside the row
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    if (jj < nt) {
                        const float zv = bf16_bits_to_float(zt[jj * 128]);
                        op[(size_t)jj * p.Vh * 128] = float_to_bf16_bits(o[jj] * rs[jj] * wn * silu_f(zv));
                    }
                }
            }
            named_barrier_sync(3, kEThreads);
            if (et == 0) {
                if (full) {
                    tma_store_2d(&tmO, smem + OFF_Z, h * 128, tok0);
                    bulk_commit();
                }
                if (c + 1 < nchunks) {
                    bulk_wait_read_all();  // the output tile has left shared memory
                    load_z(c + 1);
                }
            }
            __syncwarp();
        }
        if (et == 0) bulk_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn
