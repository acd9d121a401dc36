// Chunked prefill of the gated delta rule on 5th-generation tensor cores:
// the state recurrence over the chunks of a row, and the gated-RMSNorm output.
//
// The recurrence (Qwen3.8 27B model card, "Gated DeltaNet" bullet), per value
// head with state S [128 v][128 k]:
//     S_t = exp(g_t) S_{t-1} + u_t k_t^T,   u_t = beta_t (v_t - exp(g_t) S_{t-1} k_t),
//     o_t = S_t q_t.
// Over a chunk of 64 tokens, with the per-chunk record of wy.cuh (T1, W, M and
// the decays, none of which depends on the state):
//     U   = T1 V - W S0^T                                   (U~ = T1 V)
//     O   = Qs S0^T + M U                                   (Qs = diag(e^G) Q)
//     S_C = e^{G_C} S0 + U^T K'                             (K' = diag(e^{G_C - G}) K).
//
// One CTA owns one (row, value head) and walks its chunks in order.  Per chunk
// the tensor cores run four products, all tcgen05.mma kind::f16 with M = 128
// and f32 accumulators in TMEM:
//     MMA-P  U~^T        = V^T T1^T                 (state-free, issued a chunk ahead)
//     MMA-A  [U^T | O^T] += S0 [-W ; Qs]^T           (one N = 128 pass; S0 as f16 in TMEM)
//     MMA-S  S           += U^T K'                   (U^T as f16 in TMEM)
//     MMA7   O^T         += U^T M^T
// Only MMA-A, the f16 conversion of U^T, MMA-S and the f16 copy of the new
// state are on the sequential path from one chunk to the next; a single
// issuing thread keeps the tensor pipe fed while
//   * the converters (8 warps) turn U^T and the state into f16 operands, then
//     scale the f32 state by the next chunk's e^{G_C} while MMA-A runs,
//   * the preparers (4 warps) scale the Q and K tiles of the next chunk in
//     shared memory into Qs and K' (the decays come with the record), and
//   * the epilogue (16 warps, 16 tokens each) turns O^T of chunk c into the
//     gated RMSNorm and the bf16 output while the chain is on chunk c+1 (two
//     accumulators).
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
    int c0, c1;               // chunk window [c0, c1) of every row (c1 < 0: to the end of the row)
    const int* slots;         // [N] state row of each packed row (validated by the host), or nullptr
    const int* order;         // [N] packed row of each grid row (longest first), or nullptr: grid row = row
    int rec_chunks;           // chunks the record array holds  } the index checks of
    int state_rows;           // rows of the state arrays       } the debug build
};

namespace chunk {
constexpr int C = 64;              // tokens per chunk
constexpr int kCThreads = 256;     // converters, warps 0-7
constexpr int kEThreads = 512;     // epilogue, warps 8-23
constexpr int kPThreads = 128;     // preparers, warps 24-27
constexpr int kIssuerWarp = 28;    // tensor-core issue
constexpr int kLoaderWarp = 29;    // TMA loads of the chunk inputs
constexpr int kThreads = kCThreads + kEThreads + kPThreads + 64;
// one input buffer; every tile is f16 [64 rows][64] with 128-byte rows in the TMA 128B swizzle
constexpr uint32_t BUF_V = 0;        // V [t][v], 2 column blocks (TMA)
constexpr uint32_t BUF_T1 = 16384;   // T1 (record)
constexpr uint32_t BUF_WQ = 24576;   // per k block b at 16384 b: -W (record), then Q (TMA) scaled in place to Qs
constexpr uint32_t BUF_M = 57344;    // M (record)
constexpr uint32_t BUF_KP = 65536;   // K (TMA), 2 column blocks, scaled in place to K'
constexpr uint32_t BUF_DEC = 81920;  // f32 e^{G_C - G_t} [64], e^{G_t} [64], e^{G_C} (record)
constexpr uint32_t BUF_BYTES = 82944;  // rounded up to 1 KB
static_assert(BUF_DEC + wy::REC_DEC_BYTES <= BUF_BYTES, "input buffer");
// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_BUF0 = 0;
constexpr uint32_t OFF_BUF1 = BUF_BYTES;
constexpr uint32_t OFF_Z = 2 * BUF_BYTES;  // 2 x z bf16 [64 t][128], plain row-major; the output tiles
constexpr uint32_t OFF_MISC = OFF_Z + 2 * 16384;
constexpr uint32_t MISC_BYTES = 2048;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
// misc: 0 barriers, 256 TMEM slot, 512 reductions [4][64], 1536 rstd [64]
// TMEM columns (32-bit, 128 lanes = v rows)
constexpr uint32_t T_S = 0;                  // state f32 [128 v][128 k]
constexpr uint32_t T_D0 = 128, T_D1 = 256;   // per buffer: U^T f32 [128][64] at +0, O^T at +64
constexpr uint32_t T_S16 = 384;              // state f16, k pairs (A of MMA-A)
constexpr uint32_t T_U16 = 448;              // U^T f16, t pairs (A of MMA-S and MMA7)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t LD_BYTES = 3 * 16384 + 4 * 8192 + wy::REC_DEC_BYTES;
constexpr uint32_t Z_BYTES = 64 * 128 * 2;
constexpr uint32_t ID_P = idesc_f16_f32(128, 64, true, false, false);   // V^T (MN-major) x T1 (K-major)
constexpr uint32_t ID_A = idesc_f16_f32(128, 128, false, false, false); // S16 x [-W ; Qs] (K-major)
constexpr uint32_t ID_S = idesc_f16_f32(128, 128, false, true, false);  // U16 x K' (MN-major)
constexpr uint32_t ID_7 = idesc_f16_f32(128, 64, false, false, false);  // Up x M (K-major)
// mbarrier slots
constexpr int B_LD = 0;     // + buffer: inputs landed
constexpr int B_A = 2;      // MMA-A complete
constexpr int B_UC = 3;     // U^T converted (one arrive per converter warp)
constexpr int B_SM = 4;     // MMA-S complete
constexpr int B_SC = 5;     // state converted (one arrive per converter warp)
constexpr int B_O = 6;      // + buffer: MMA7 complete, O^T final
constexpr int B_E = 8;      // + buffer: the epilogue has read and cleared O^T
constexpr int B_FREE = 10;  // + buffer: every MMA that reads the buffer is complete
constexpr int B_Z = 12;     // + z buffer: z tile landed
constexpr int B_SS = 14;    // f32 state scaled by e^{G_C} (one arrive per converter warp)
constexpr int B_PREP = 15;  // + buffer: Qs and K' ready (one arrive per preparer warp)
constexpr int kBars = 17;
static_assert(SMEM_BYTES <= 232448, "shared memory");
}  // namespace chunk

__global__ void __launch_bounds__(chunk::kThreads, 1)
    gdn_chunk_kernel(const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmO,
                     const ChunkParams p) {
    using namespace chunk;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int h = blockIdx.x;
    const int n = p.order ? __ldg(p.order + blockIdx.y) : (int)blockIdx.y;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int kap = h / (p.Vh / p.Kh);
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int hf = (warp >> 2) & 1;           // column half within the group
    const int row = 32 * q4 + lane;           // v row of the state / output channel
    const uint32_t tlane = (static_cast<uint32_t>(32 * q4) << 16);

    uint8_t* misc = smem + OFF_MISC;
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(misc + 256);
    float* s_red = reinterpret_cast<float*>(misc + 512);    // [4][64]
    float* s_rstd = reinterpret_cast<float*>(misc + 1536);  // [64]

    int start, len;
    p.seq.bounds(n, start, len);
    const int srow = p.slots ? __ldg(p.slots + n) : n;  // state row
    // the chunks [cw, cw + nchunks) of the row; loop indices below count from cw
    const int cw = min(p.c0, (len + C - 1) / C);
    const int nchunks = max(0, (p.c1 < 0 ? (len + C - 1) / C : min(p.c1, (len + C - 1) / C)) - cw);
    const int cbase = (p.chunk_base ? __ldg(p.chunk_base + n) : n * ((p.seq.uniform_T + C - 1) / C)) + cw;
    start += cw * C;
    len -= cw * C;

    if (tid == 0) {
        for (int i = 0; i < kBars; ++i)
            mbar_init(&bars[i], (i == B_UC || i == B_SC || i == B_SS) ? kCThreads / 32
                                : (i == B_PREP || i == B_PREP + 1) ? kPThreads / 32
                                                                   : 1);
        fence_barrier_init();
        prefetch_tensormap(&tmV);
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
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
    auto dacc = [&](int c) { return tbase + ((c & 1) ? T_D1 : T_D0); };
    // (debug build: a record index out of range is recorded and record 0 is read instead)
    auto rec_of = [&](int c) {
        const bool ok = GDN_CHECK(cbase + c >= 0 && cbase + c < p.rec_chunks);
        return p.rec + (ok ? ((size_t)(cbase + c) * p.Vh + h) * wy::REC_BYTES : 0);
    };
    auto load_chunk = [&](int c) {
        uint8_t* B = buf(c);
        uint64_t* bar = &bars[B_LD + (c & 1)];
        const int y = start + c * C;
        (void)GDN_CHECK(y >= 0 && y < p.total);
        mbar_arrive_expect_tx(bar, LD_BYTES);
        tma_load_2d(B + BUF_V, &tmV, h * 128, y, bar);
        tma_load_2d(B + BUF_V + 8192, &tmV, h * 128 + 64, y, bar);
        tma_load_2d(B + BUF_WQ + 8192, &tmQ, kap * 128, y, bar);
        tma_load_2d(B + BUF_WQ + 24576, &tmQ, kap * 128 + 64, y, bar);
        tma_load_2d(B + BUF_KP, &tmK, kap * 128, y, bar);
        tma_load_2d(B + BUF_KP + 8192, &tmK, kap * 128 + 64, y, bar);
        const uint8_t* r = rec_of(c);
        bulk_load(B + BUF_T1, r + wy::REC_T1, 8192, bar);
        bulk_load(B + BUF_WQ, r + wy::REC_MW, 8192, bar);
        bulk_load(B + BUF_WQ + 16384, r + wy::REC_MW + 8192, 8192, bar);
        bulk_load(B + BUF_M, r + wy::REC_M, 8192, bar);
        bulk_load(B + BUF_DEC, r + wy::REC_DEC, wy::REC_DEC_BYTES, bar);
    };
    auto prefetch_chunk = [&](int c) {
        const int y = start + c * C;
        prefetch_tma_2d(&tmV, h * 128, y);
        prefetch_tma_2d(&tmV, h * 128 + 64, y);
        prefetch_tma_2d(&tmQ, kap * 128, y);
        prefetch_tma_2d(&tmQ, kap * 128 + 64, y);
        prefetch_tma_2d(&tmK, kap * 128, y);
        prefetch_tma_2d(&tmK, kap * 128 + 64, y);
        prefetch_l2(rec_of(c), wy::REC_BYTES);
    };
    auto load_z = [&](int c) {
        uint64_t* bar = &bars[B_Z + (c & 1)];
        mbar_arrive_expect_tx(bar, Z_BYTES);
        tma_load_2d(smem + OFF_Z + (c & 1) * 16384, &tmZ, h * 128, start + c * C, bar);
    };
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

    if (warp == kIssuerWarp) {
        // =================================================================== issue
        if (lane == 0 && nchunks > 0) {
            // MMA-P: U~^T of chunk c into the U^T half of its accumulator
            auto mma_P = [&](int c) {
                const uint32_t B = smem_u32(buf(c));
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16(dacc(c), sw128_desc(B + BUF_V + s * 2048, 8192, 1024),
                            sw128_desc(B + BUF_T1 + s * 32, 16, 1024), ID_P, s > 0);
            };
            wait1(B_LD, 0);
            tc_fence_after();
            mma_P(0);
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                const uint32_t B = smem_u32(buf(c));
                const uint32_t d = dacc(c);
                wait1(B_E + b, (c >> 1) & 1);  // O^T[b] cleared
                wait1(B_SC, c & 1);            // state of chunk c in f16
                wait1(B_PREP + b, (c >> 1) & 1);  // Qs and K' of chunk c
                tc_fence_after();
                // MMA-A: [U^T | O^T] += S0 [-W ; Qs]^T
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_f16_ta(d, tbase + T_S16 + 8 * s,
                               sw128_desc(B + BUF_WQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024), ID_A,
                               1);
                mma_commit(&bars[B_A]);
                // U~ of the next chunk now if its inputs are in, else after MMA7
                bool p_next = c + 1 < nchunks;
                if (p_next && mbar_try_wait(smem_u32(&bars[B_LD + (b ^ 1)]), ((c + 1) >> 1) & 1)) {
                    tc_fence_after();
                    mma_P(c + 1);
                    p_next = false;
                }
                wait1(B_UC, c & 1);
                wait1(B_SS, c & 1);  // f32 state scaled by e^{G_C} of chunk c
                tc_fence_after();
                // MMA-S: S += U^T K'
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(tbase + T_S, tbase + T_U16 + 8 * s,
                               sw128_desc(B + BUF_KP + s * 2048, 8192, 1024), ID_S, 1);
                mma_commit(&bars[B_SM]);
                // MMA7: O^T += U^T M^T
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_f16_ta(d + 64, tbase + T_U16 + 8 * s,
                               sw128_desc(B + BUF_M + s * 32, 16, 1024), ID_7, 1);
                mma_commit(&bars[B_O + b]);
                mma_commit(&bars[B_FREE + b]);
                if (p_next) {
                    wait1(B_LD + (b ^ 1), ((c + 1) >> 1) & 1);
                    tc_fence_after();
                    mma_P(c + 1);
                }
            }
        }
        __syncwarp();
    } else if (warp == kLoaderWarp) {
        // =================================================================== loads
        if (lane == 0 && nchunks > 0) {
            load_chunk(0);
            if (nchunks > 1) load_chunk(1);
            int issued = nchunks > 1 ? 2 : 1;  // chunks whose inputs were requested
            for (int c = 2; c < nchunks && c < 4; ++c) prefetch_chunk(c);
            // a buffer takes chunk c+2 once every MMA that reads chunk c is done
            for (int c = 0; c + 2 < nchunks; ++c) {
                wait1(B_FREE + (c & 1), (c >> 1) & 1);
                if (broken) break;  // no copy into a buffer that may still be read
                load_chunk(c + 2);
                issued = c + 3;
                if (c + 4 < nchunks) prefetch_chunk(c + 4);
            }
            // after a wait ran out, the CTA exits only once its copies in flight have landed
            // (the last request of each buffer; bounded)
            if (broken)
                for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c) mbar_wait(&bars[B_LD + (c & 1)], (c >> 1) & 1);
        }
        __syncwarp();
    } else if (tid < kCThreads) {
        // =================================================================== converters
        // initial state: f16 copy for MMA-A, f32 scaled by the first chunk's e^{G_C}
        {
            float gC = 1.f;
            if (nchunks > 0) {
                wait(B_LD, 0);
                gC = reinterpret_cast<const float*>(buf(0) + BUF_DEC)[128];
            }
            const float* src = p.init_state && GDN_CHECK(srow >= 0 && srow < p.state_rows)
                                   ? p.init_state + (((size_t)srow * p.Vh + h) * 128 + row) * 128 + 64 * hf
                                   : nullptr;
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
                uint32_t hpk[16], r[32];
#pragma unroll
                for (int j = 0; j < 16; ++j) hpk[j] = pack_half2(v[2 * j], v[2 * j + 1]);
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
                tmem_st16(tbase + tlane + T_S16 + 32 * hf + 16 * half, hpk);
                tmem_st32(tbase + tlane + T_S + 64 * hf + 32 * half, r);
            }
            tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&bars[B_SC]);
            mbar_arrive(&bars[B_SS]);
        }

        for (int c = 0; c < nchunks; ++c) {
            // ---- U^T to f16 (A of MMA-S and MMA7)
            wait(B_A, c & 1);
            tc_fence_after();
            {
                float u[32];
                tmem_ld32(dacc(c) + tlane + 32 * hf, u);
                tmem_ld_wait();
                uint32_t up[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) up[j] = pack_half2(u[2 * j], u[2 * j + 1]);
                tmem_st16(tbase + tlane + T_U16 + 16 * hf, up);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_UC]);

            // ---- the new state: f16 copy for the next MMA-A first, then the f32 state
            // scaled by the next e^{G_C} (needed only by the next MMA-S)
            wait(B_SM, c & 1);
            tc_fence_after();
            if (c + 1 < nchunks) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tbase + tlane + T_S + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
                    uint32_t hpk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) hpk[j] = pack_half2(v[2 * j], v[2 * j + 1]);
                    tmem_st16(tbase + tlane + T_S16 + 32 * hf + 16 * half, hpk);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SC]);
                wait(B_LD + ((c + 1) & 1), ((c + 1) >> 1) & 1);
                const float gC = reinterpret_cast<const float*>(buf(c + 1) + BUF_DEC)[128];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float v[32];
                    tmem_ld32(tbase + tlane + T_S + 64 * hf + 32 * half, v);
                    tmem_ld_wait();
                    uint32_t r[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gC * v[j]);
                    tmem_st32(tbase + tlane + T_S + 64 * hf + 32 * half, r);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_SS]);
            }
        }

        if (!broken && p.final_state != nullptr && GDN_CHECK(srow >= 0 && srow < p.state_rows)) {
            float* dst = p.final_state + (((size_t)srow * p.Vh + h) * 128 + row) * 128 + 64 * hf;
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
    } else if (tid < kCThreads + kEThreads) {
        // =================================================================== epilogue
        const int et = tid - kCThreads;
        const int qt = (warp - 8) >> 2;                 // token quarter of this warp
        const float wn = 1.0f + __ldg(p.norm_w + row);  // (1 + w) of this thread's v channel
        const uint32_t zero[16] = {};
        // both O^T accumulators start cleared
        tmem_st16(tbase + tlane + T_D0 + 64 + 16 * qt, zero);
        tmem_st16(tbase + tlane + T_D1 + 64 + 16 * qt, zero);
        tmem_st_wait();
        tc_fence_before();
        named_barrier_sync(3, kEThreads);
        if (et == 0) {
            mbar_arrive(&bars[B_E]);
            mbar_arrive(&bars[B_E + 1]);
        }
        if (et == 32 && nchunks > 0) load_z(0);
        __syncwarp();
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int tok0 = start + c * C;
            const int nv = min(C, len - c * C);
            const uint32_t tO = dacc(c) + 64 + tlane + 16 * qt;
            // z of chunk c+1 into the other tile, once the output of chunk c-1 has left it
            // (thread 32 of the epilogue owns the output stores and z loads)
            if (et == 32 && c + 1 < nchunks) {
                bulk_wait_read_all();
                load_z(c + 1);
            }
            __syncwarp();
            wait(B_O + b, (c >> 1) & 1);
            tc_fence_after();
            float o[16];
            tmem_ld16(tO, o);
            tmem_ld_wait();
            tmem_st16(tO, zero);  // cleared for chunk c+2
            tmem_st_wait();
            tc_fence_before();
            {
                float sq[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) sq[jj] = o[jj] * o[jj];
                const float part = warp_transpose_sum16(sq, lane);  // token lane >> 1
                if ((lane & 1) == 0) s_red[q4 * 64 + 16 * qt + (lane >> 1)] = part;
            }
            named_barrier_sync(3, kEThreads);
            if (et == 0) mbar_arrive(&bars[B_E + b]);  // O^T[b] may take chunk c+2
            if (et < 64)
                s_rstd[et] = rsqrtf((s_red[et] + s_red[64 + et] + s_red[128 + et] + s_red[192 + et]) * (1.0f / 128.0f) +
                                    kEps);
            named_barrier_sync(3, kEThreads);
            wait(B_Z + b, (c >> 1) & 1);
            // a full chunk is written over its z tile and leaves by one TMA store; a ragged
            // last chunk is stored directly (the rows past it belong to the next sequence)
            uint16_t* zt = reinterpret_cast<uint16_t*>(smem + OFF_Z + b * 16384) + 16 * qt * 128 + row;
            const float* rs = s_rstd + 16 * qt;
            {
                float zv[16];
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) zv[jj] = bf16_bits_to_float(zt[jj * 128]);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) o[jj] = o[jj] * rs[jj] * wn * silu_tanh(zv[jj]);
            }
            // bf16 rounding two tokens at a time (one paired conversion)
            uint32_t yb[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) yb[j] = pack_bf16x2(o[2 * j], o[2 * j + 1]);
            const bool full = (nv == C);
            if (full) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    zt[(2 * j) * 128] = static_cast<uint16_t>(yb[j]);
                    zt[(2 * j + 1) * 128] = static_cast<uint16_t>(yb[j] >> 16);
                }
                fence_proxy_async_smem();
            } else {
                uint16_t* op = p.out + (size_t)(tok0 + 16 * qt) * p.Vh * 128 + h * 128 + row;
                const int nt = nv - 16 * qt;  // tokens of this quarter inside the row
#pragma unroll
                for (int jj = 0; jj < 16; ++jj)
                    if (jj < nt && GDN_CHECK(tok0 + 16 * qt + jj < p.total))
                        op[(size_t)jj * p.Vh * 128] = static_cast<uint16_t>((jj & 1) ? (yb[jj >> 1] >> 16) : yb[jj >> 1]);
            }
            named_barrier_sync(3, kEThreads);
            if (et == 32 && full) {
                tma_store_2d(&tmO, smem + OFF_Z + b * 16384, h * 128, tok0);
                bulk_commit();
            }
            __syncwarp();
        }
        if (et == 32) {
            bulk_wait_all();
            // after a wait ran out, the z tiles in flight land before the CTA exits (bounded)
            if (broken)
                for (int k = nchunks > 2 ? nchunks - 2 : 0; k < nchunks; ++k) mbar_wait(&bars[B_Z + (k & 1)], (k >> 1) & 1);
        }
    } else {
        // =================================================================== preparers
        // Qs = diag(e^G) Q and K' = diag(e^{G_C - G}) K, in place; one row of 64 k per thread per block
        const int pt = tid - (kCThreads + kEThreads);
        const int which = pt >> 6;  // 0: Q rows, 1: K rows
        const int t = pt & 63;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            wait(B_LD + b, (c >> 1) & 1);
            uint8_t* B = buf(c);
            const float sc = reinterpret_cast<const float*>(B + BUF_DEC)[which ? t : 64 + t];
#pragma unroll
            for (int blk = 0; blk < 2; ++blk) {
                uint8_t* tile = which ? B + BUF_KP + blk * 8192 : B + BUF_WQ + 8192 + blk * 16384;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint4* q = reinterpret_cast<uint4*>(tile + sw128_chunk(t, cc));
                    uint4 v = *q;
                    uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[e]));
                        u[e] = pack_half2(f.x * sc, f.y * sc);
                    }
                    *q = v;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_PREP + b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace gdn
