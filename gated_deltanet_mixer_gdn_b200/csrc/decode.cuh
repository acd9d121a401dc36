// Decode of the Gated DeltaNet mixer: one token (or k successive tokens) for
// each of `rows` rows.
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
// once.  With k tokens per row (speculative verification, several tokens per
// call) each state row stays in registers through the k sequential updates:
// the state is still read and written once per call, k tokens at a time.
//
// Work item = (row, q/k head): the conv of the q/k head's 256 channels and of
// its value heads' 128-channel slices, the L2 norms and gates, then the states
// of those value heads.  Every conv-history channel therefore has exactly one
// reader and writer, and the in-place history shift needs no cross-CTA sync.
// Persistent CTAs (one per SM) walk items round-robin.  A producer warp
// streams each state in 32 KiB half-tiles (64 state rows) with bulk copies
// into a ring of shared-memory stages, running up to a full item ahead; a
// group of eight compute warps reads a half-tile (8 rows per warp: each lane
// holds 16 columns of 2 rows, eight lanes reading 128 contiguous bytes), sums
// each row's two dot products over its eight lanes with one transposed
// shuffle reduction, and writes the updated rows straight back to HBM with
// coalesced 128-bit stores.  With several tokens per row two such groups take
// alternate items, so that one group's conv, norms and output overlap the
// other's state stream.
#pragma once

#include "common.cuh"

#ifndef GDN_DECODE_STAGES
#define GDN_DECODE_STAGES 5
#endif

namespace gdn {

struct DecodeParams {
    int Kh, Vh, C, rows, nitems;
    int ntok;                // tokens per row (1 .. the kernel's maximum)
    const uint16_t* qkv;     // bf16 [rows][ntok][C]
    const uint16_t* z;       // bf16 [rows][ntok][Vh*128]
    const uint16_t* a;       // bf16 [rows][ntok][Vh]
    const uint16_t* b;       // bf16 [rows][ntok][Vh]
    const uint16_t* conv_w;  // bf16 [C][4]
    const float* A_log;      // [Vh]
    const float* dt_bias;    // [Vh]
    const float* norm_w;     // [128]
    float* state;            // f32 [rows or pool][Vh][128][128], in place
    float* conv;             // f32 [rows or pool][3][C], in place
    uint16_t* out;           // bf16 [rows][ntok][Vh*128]
    const int* slots;        // [rows] state / history row of each batch row (validated by the host), or nullptr
    int pool_rows;           // rows of the state and history arrays (the index checks of the debug build)
};

// State and history row of batch row r (debug build: a row out of range is recorded and row
// 0 is used instead).
__device__ __forceinline__ int decode_slot(const DecodeParams& p, int r) {
    const int s = p.slots ? __ldg(p.slots + r) : r;
    return GDN_CHECK(r >= 0 && r < p.rows && s >= 0 && s < p.pool_rows) ? s : 0;
}

namespace dec {
constexpr int kMaxStages = GDN_DECODE_STAGES;
constexpr int kMaxGroup = 8;                     // value heads per q/k head (Vh / Kh)
constexpr uint32_t kTileBytes = 64 * 128 * 4;   // half of a head's state
constexpr int kComputeThreads = 256;            // one group of compute warps
// Groups of compute warps: with several tokens per row, two groups take alternate items, so
// that one group's conv, norms and output of an item overlap the other's state stream.
__host__ __device__ constexpr int groups(int kmax) { return kmax > 1 ? 2 : 1; }
__host__ __device__ constexpr int threads(int kmax) { return groups(kmax) * kComputeThreads + 32; }  // + producer
constexpr int kSlots = (2 + kMaxGroup) * 128 / kComputeThreads;  // conv channels per thread (max)
constexpr uint32_t kSmemLimit = 232448;         // opt-in shared memory per block on sm_100
constexpr int kMaxTokens = 8;                   // tokens per row of the multi-token kernel

// Shared-memory plan for a group size G and n tokens per row: a ring of
// half-tile stages, then two buffers of per-item inputs, bulk-copied one item
// ahead (history [3][(2+G)*128] f32, new qkv [n][(2+G)*128] bf16, conv taps
// [(2+G)*128][4] bf16, z [n][G*128] bf16), then scratch: barriers (256 B),
// q, k [n][128], v, o [n][G][128], reductions [n][8 + 8G], gates [n][G][2], k.q [n].
struct Plan {
    int stages;
    uint32_t aux_x, aux_w, aux_z, aux_bytes, aux_load_bytes, off_aux, off_misc, misc_bytes, smem_bytes;
    uint32_t m_q, m_k, m_v, m_o, m_red, m_gate;  // float offsets of the scratch arrays (from off_misc + 256)
    uint32_t group_floats;                        // scratch of one group of compute warps
};
__host__ __device__ inline Plan plan(int G, int n, int ngroups) {
    Plan pl{};
    const uint32_t nch = (2 + G) * 128;
    pl.aux_x = 3 * nch * 4;
    pl.aux_w = pl.aux_x + n * nch * 2;
    pl.aux_z = pl.aux_w + nch * 8;
    pl.aux_load_bytes = pl.aux_z + n * G * 256;
    pl.aux_bytes = (pl.aux_load_bytes + 127) / 128 * 128;
    pl.m_q = 0;
    pl.m_k = pl.m_q + n * 128;
    pl.m_v = pl.m_k + n * 128;
    pl.m_o = pl.m_v + n * G * 128;
    pl.m_red = pl.m_o + n * G * 128;
    pl.m_gate = pl.m_red + n * (8 + 8 * G);
    pl.group_floats = (pl.m_gate + n * G * 2 + n + 31) / 32 * 32;  // gates, then k.q [n]
    pl.misc_bytes = 256 + ngroups * pl.group_floats * 4;
    const uint32_t rest = 2 * pl.aux_bytes + pl.misc_bytes + 1024;
    int st = (int)((kSmemLimit - rest) / kTileBytes);
    pl.stages = st > kMaxStages ? kMaxStages : st;
    pl.off_aux = pl.stages * kTileBytes;
    pl.off_misc = pl.off_aux + 2 * pl.aux_bytes;
    pl.smem_bytes = pl.off_misc + pl.misc_bytes + 1024;
    return pl;
}
}  // namespace dec

// The row arithmetic, with every fused multiply-add written out, so that the one-token and
// the several-token kernels round identically whatever the compiler would contract.
__device__ __forceinline__ float dot4(const float4 a, const float4 b) {
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, a.x * b.x)));
}
// sum of the products of 16 columns (4 chunks of 4), in a fixed order
__device__ __forceinline__ float dot16(const float4 (&a)[4], const float4 (&b)[4]) {
    float acc = a[0].x * b[0].x;
    acc = fmaf(a[0].y, b[0].y, acc);
    acc = fmaf(a[0].z, b[0].z, acc);
    acc = fmaf(a[0].w, b[0].w, acc);
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        acc = fmaf(a[i].x, b[i].x, acc);
        acc = fmaf(a[i].y, b[i].y, acc);
        acc = fmaf(a[i].z, b[i].z, acc);
        acc = fmaf(a[i].w, b[i].w, acc);
    }
    return acc;
}
// Four values per lane, summed over each aligned group of 8 lanes: lane l ends with the sum of
// value ((l >> 2) & 1) * 2 + ((l >> 1) & 1).
__device__ __forceinline__ float group8_transpose_sum4(const float (&v)[4], int lane) {
    const bool up4 = (lane & 4) != 0;
    const float w0 = (up4 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, up4 ? v[0] : v[2], 4);
    const float w1 = (up4 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, up4 ? v[1] : v[3], 4);
    const bool up2 = (lane & 2) != 0;
    const float x = (up2 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, up2 ? w0 : w1, 2);
    return x + __shfl_xor_sync(0xffffffffu, x, 1);
}
// alpha s + u k
__device__ __forceinline__ float4 decay_add(const float4 s, float alpha, float u, const float4 k) {
    return make_float4(fmaf(u, k.x, alpha * s.x), fmaf(u, k.y, alpha * s.y), fmaf(u, k.z, alpha * s.z),
                       fmaf(u, k.w, alpha * s.w));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Once one of this thread's waits has run out (`broken`), it waits no more: it records
// the error once, and the caller no longer releases buffers or issues copies.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, bool& broken) {
    if (broken) return false;
    if (!mbar_wait_for(bar, parity, g_decode_wait_limit_ns)) {
        broken = true;
        record_error(kErrTimeoutTma);
        return false;
    }
    return true;
}

// SPLIT = false: an item is a q/k group (all its value heads), persistent CTAs walk the items.
// SPLIT = true: an item is one value head; the Vh / Kh items of a group are the CTAs of one
// thread-block cluster (one item each), launched with that cluster size.
template <int KMAX, bool SPLIT>
__global__ void __launch_bounds__(dec::threads(KMAX), 1) gdn_decode_kernel(const DecodeParams p) {
    using namespace dec;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int Gfull = p.Vh / p.Kh;         // value heads per q/k head
    const int G = SPLIT ? 1 : Gfull;       // value heads of one item
    const int ns = SPLIT ? Gfull : 1;      // items per q/k group
    const int nt = KMAX == 1 ? 1 : p.ntok;  // tokens per row
    constexpr int NG = groups(KMAX);
    const Plan pl = plan(G, nt, NG);
    const int nst = pl.stages;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + pl.off_misc);
    uint64_t* empty = full + kMaxStages;
    uint64_t* auxfull = empty + kMaxStages;
    uint64_t* auxempty = auxfull + 2;
    uint64_t* qkfree = auxempty + 2;  // split groups: the peers have read the q/k history (rank 0's copy)
    float* scratch = reinterpret_cast<float*>(smem + pl.off_misc + 256);
    float* s_q = scratch + pl.m_q;        // [nt][128]
    float* s_k = scratch + pl.m_k;        // [nt][128]
    float* s_v = scratch + pl.m_v;        // [nt][G][128]
    float* s_o = scratch + pl.m_o;        // [nt][G][128]
    float* s_red = scratch + pl.m_red;    // [nt][8 + 8G]
    float* s_gate = scratch + pl.m_gate;  // [nt][G][2], then k.q [nt]
    float* s_kq = s_gate + nt * G * 2;
    const int nred = 8 + 8 * G;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int nch = (2 + G) * 128;  // conv channels of one item: q, k, then G value slices
    const int units_per_item = 2 * G;
    const int nmine = (p.nitems > (int)blockIdx.x) ? (p.nitems - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const int nunits = nmine * units_per_item;
    bool broken = false;

    if (tid == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kComputeThreads / 32);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&auxfull[s], 1);
            mbar_init(&auxempty[s], kComputeThreads / 32);
        }
        if (SPLIT) mbar_init(qkfree, ns - 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (SPLIT) cluster_sync();  // the cluster's barriers are initialised before any remote arrive

    // item it -> batch row, q/k head, first value head (within the group) of the item
    auto item = [&](int it, int& row, int& kap, int& hoff) {
        const int rk = SPLIT ? it / ns : it;
        row = rk / p.Kh;
        kap = rk - row * p.Kh;
        hoff = SPLIT ? it - rk * ns : 0;
    };

    // unit u of this CTA: item u / (2G), value head (u % 2G) / 2 of its group, half u % 2
    auto unit_ptr = [&](int u) -> float* {
        int row, kap, hoff;
        item(blockIdx.x + (u / units_per_item) * gridDim.x, row, kap, hoff);
        const int r = u % units_per_item;
        const int head = kap * Gfull + hoff + (r >> 1);
        return p.state + (((size_t)decode_slot(p, row) * p.Vh + head) * 128 + (r & 1) * 64) * 128;
    };

    if (warp == NG * kComputeThreads / 32) {
        // ---------------- producer warp: per-item inputs one item ahead, state half-tiles in a ring
        if (lane == 0) {
            auto aux_load = [&](int m) {
                int row, kap, hoff;
                item(blockIdx.x + m * gridDim.x, row, kap, hoff);
                uint8_t* ax = smem + pl.off_aux + (m & 1) * pl.aux_bytes;
                uint64_t* bar = &auxfull[m & 1];
                mbar_arrive_expect_tx(bar, pl.aux_load_bytes);
                const int chq = kap * 128, chk = p.Kh * 128 + kap * 128, chv = 2 * p.Kh * 128 + (kap * Gfull + hoff) * 128;
                const int srow = decode_slot(p, row);
                for (int r = 0; r < 3; ++r) {
                    const float* hrow = p.conv + ((size_t)srow * 3 + r) * p.C;
                    float* dst = reinterpret_cast<float*>(ax) + r * nch;
                    bulk_load(dst, hrow + chq, 512, bar);
                    bulk_load(dst + 128, hrow + chk, 512, bar);
                    bulk_load(dst + 256, hrow + chv, G * 512, bar);
                }
                for (int j = 0; j < nt; ++j) {
                    const uint16_t* xrow = p.qkv + ((size_t)row * nt + j) * p.C;
                    uint16_t* dx = reinterpret_cast<uint16_t*>(ax + pl.aux_x) + j * nch;
                    bulk_load(dx, xrow + chq, 256, bar);
                    bulk_load(dx + 128, xrow + chk, 256, bar);
                    bulk_load(dx + 256, xrow + chv, G * 256, bar);
                    bulk_load(ax + pl.aux_z + j * G * 256,
                              p.z + (((size_t)row * nt + j) * p.Vh + kap * Gfull + hoff) * 128, G * 256, bar);
                }
                uint16_t* dw = reinterpret_cast<uint16_t*>(ax + pl.aux_w);
                bulk_load(dw, p.conv_w + (size_t)chq * 4, 1024, bar);
                bulk_load(dw + 512, p.conv_w + (size_t)chk * 4, 1024, bar);
                bulk_load(dw + 1024, p.conv_w + (size_t)chv * 4, G * 1024, bar);
            };
            // the next item's inputs are requested once the ring holds this item's first stages,
            // by which time the item two back has released their buffer.  A buffer is only
            // refilled after every consumer released it, so no phase is armed twice; if a wait
            // for a release runs out (the consumers stopped releasing after a wait of their own
            // ran out), no further copy is issued.
            const int lead = nst < units_per_item - 1 ? nst : units_per_item - 1;
            const int stop_at = g_decode_stop_copies_at;  // test hook, -1 normally
            int issued = 0, issued_aux = 0;
            if (nmine > 0) {
                aux_load(0);
                issued_aux = 1;
            }
            for (int u = 0; u < nunits; ++u) {
                const int m = u / units_per_item, r = u % units_per_item;
                if (r == lead && m + 1 < nmine) {
                    if (m >= 1 && !bounded_wait(&auxempty[(m + 1) & 1], ((m - 1) >> 1) & 1, broken)) break;
                    aux_load(m + 1);
                    issued_aux = m + 2;
                }
                const int st = u % nst;
                if (u == stop_at) break;
                if (u >= nst && !bounded_wait(&empty[st], ((u / nst) - 1) & 1, broken)) break;
                mbar_arrive_expect_tx(&full[st], kTileBytes);
                bulk_load(smem + st * kTileBytes, unit_ptr(u), kTileBytes, &full[st]);
                issued = u + 1;
            }
            // Drain: every copy issued into this CTA's shared memory has landed before the CTA
            // can exit (on the normal path these phases are complete already).  Only the last
            // phase armed on each buffer can still be open.
            for (int v = issued > nst ? issued - nst : 0; v < issued; ++v)
                mbar_wait(&full[v % nst], (v / nst) & 1);
            for (int m = issued_aux > 2 ? issued_aux - 2 : 0; m < issued_aux; ++m)
                mbar_wait(&auxfull[m & 1], (m >> 1) & 1);
        }
        return;
    }

    // ---------------- compute warps: group cg of NG takes this CTA's items cg, cg + NG, ...
    const int cg = warp / (kComputeThreads / 32);
    const int ctid = tid - cg * kComputeThreads, cwarp = ctid >> 5;
    const uint32_t gbar = 1 + cg;  // named barrier of the group
    s_q += cg * pl.group_floats;
    s_k += cg * pl.group_floats;
    s_v += cg * pl.group_floats;
    s_o += cg * pl.group_floats;
    s_red += cg * pl.group_floats;
    s_gate += cg * pl.group_floats;
    s_kq += cg * pl.group_floats;
    const float w_n = (ctid < 128) ? 1.0f + p.norm_w[ctid] : 0.f;
    // gate inputs of the next item, loaded one item ahead (thread ctid < G * nt: token ctid / G, head ctid % G)
    float ga = 0.f, gb = 0.f, gA = 0.f, gdt = 0.f;
    auto gate_prefetch = [&](int m) {
        int row, kap, hoff;
        item(blockIdx.x + m * gridDim.x, row, kap, hoff);
        const int head = kap * Gfull + hoff + ctid % G, j = ctid / G;
        ga = bf16_bits_to_float(p.a[((size_t)row * nt + j) * p.Vh + head]);
        gb = bf16_bits_to_float(p.b[((size_t)row * nt + j) * p.Vh + head]);
        gA = p.A_log[head];
        gdt = p.dt_bias[head];
    };
    if (ctid < G * nt && cg < nmine) gate_prefetch(cg);
    for (int m = cg; m < nmine; m += NG) {
        int u = m * units_per_item;  // first state unit of the item
        int row, kap, hoff;
        item(blockIdx.x + m * gridDim.x, row, kap, hoff);
        const int srow = decode_slot(p, row);
        const uint8_t* ax = smem + pl.off_aux + (m & 1) * pl.aux_bytes;
        named_barrier_sync(gbar, kComputeThreads);  // previous item's readers of the scratch are done
        bounded_wait(&auxfull[m & 1], (m >> 1) & 1, broken);
        // split group: the q/k history is shifted by the group's first CTA once the others hold it
        const bool qk_writer = !SPLIT || hoff == 0;
        if (SPLIT && hoff != 0 && ctid == 0) mbar_arrive_remote(qkfree, 0);

        // ---- conv + silu of the item's channels over the nt tokens; shift their history in place
        const float* ah = reinterpret_cast<const float*>(ax);
        const uint16_t* axx = reinterpret_cast<const uint16_t*>(ax + pl.aux_x);
        const uint2* aw = reinterpret_cast<const uint2*>(ax + pl.aux_w);
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
            const int idx = ctid + s * kComputeThreads;
            if (idx < nch) {
                const int grp = idx >> 7, c = idx & 127;
                const int ch = (grp == 0) ? kap * 128 + c
                             : (grp == 1) ? p.Kh * 128 + kap * 128 + c
                                          : 2 * p.Kh * 128 + (kap * Gfull + hoff + grp - 2) * 128 + c;
                float h0 = ah[idx], h1 = ah[nch + idx], h2 = ah[2 * nch + idx];
                const uint2 wb = aw[idx];
                const float t0 = __uint_as_float(wb.x << 16), t1 = __uint_as_float(wb.x & 0xffff0000u);
                const float t2 = __uint_as_float(wb.y << 16), t3 = __uint_as_float(wb.y & 0xffff0000u);
#pragma unroll 1
                for (int j = 0; j < nt; ++j) {
                    {
                        const float x = bf16_bits_to_float(axx[j * nch + idx]);
                        const float act = silu_f(t0 * h0 + t1 * h1 + t2 * h2 + t3 * x);
                        if (grp == 0) s_q[j * 128 + c] = act;
                        else if (grp == 1) s_k[j * 128 + c] = act;
                        else s_v[(j * G + grp - 2) * 128 + c] = act;
                        h0 = h1;
                        h1 = h2;
                        h2 = x;
                    }
                }
                if (grp >= 2 || qk_writer) {
                    if (SPLIT && grp < 2) {
                        bounded_wait(qkfree, 0, broken);
                        fence_acq_rel_cluster();
                    }
                    float* hr = p.conv + (size_t)srow * 3 * p.C + ch;
                    hr[0] = h0;
                    hr[p.C] = h1;
                    hr[2 * p.C] = h2;
                }
            }
        }
        if (ctid < G * nt) {
            s_gate[2 * ctid] = expf(-expf(gA) * softplus_f(ga + gdt));  // alpha of (token ctid / G, head ctid % G)
            s_gate[2 * ctid + 1] = sigmoid_f(gb);                        // beta
            if (m + NG < nmine) gate_prefetch(m + NG);
        }
        named_barrier_sync(gbar, kComputeThreads);
        // ---- L2 norms per token: q in warps 0-3, k in warps 4-7
#pragma unroll 1
        for (int j = 0; j < nt; ++j) {
            {
                const float x = (ctid < 128) ? s_q[j * 128 + ctid] : s_k[j * 128 + ctid - 128];
                const float ss = warp_sum(x * x);
                if (lane == 0) s_red[j * nred + cwarp] = ss;
            }
        }
        named_barrier_sync(gbar, kComputeThreads);
        // q / (|q| sqrt(128)), k / |k| in place; then k.q per token (warp j of the group)
#pragma unroll 1
        for (int j = 0; j < nt; ++j) {
            {
                const float* r8 = s_red + j * nred;
                if (ctid < 128) s_q[j * 128 + ctid] *= rsqrtf(r8[0] + r8[1] + r8[2] + r8[3] + kEps) * rsqrtf(128.0f);
                else s_k[j * 128 + ctid - 128] *= rsqrtf(r8[4] + r8[5] + r8[6] + r8[7] + kEps);
            }
        }
        named_barrier_sync(gbar, kComputeThreads);
        if (cwarp < nt) {
            const float4 qf = reinterpret_cast<const float4*>(s_q + cwarp * 128)[lane];
            const float4 kf = reinterpret_cast<const float4*>(s_k + cwarp * 128)[lane];
            const float kq = warp_sum(kf.x * qf.x + kf.y * qf.y + kf.z * qf.z + kf.w * qf.w);
            if (lane == 0) s_kq[cwarp] = kq;
        }
        named_barrier_sync(gbar, kComputeThreads);

        // ---- stream the G value heads' states, two half-tiles each; nt updates per row in registers
#pragma unroll 1
        for (int hh = 0; hh < G; ++hh) {
#pragma unroll 1
            for (int half = 0; half < 2; ++half, ++u) {
                const int st = u % nst;
                bounded_wait(&full[st], (u / nst) & 1, broken);
                // the warp's 8 rows: lanes 8 g .. 8 g + 7 hold rows 2 g and 2 g + 1, lane l the
                // 16-byte column chunks (l & 7) + 8 i, i < 4 (eight lanes read 128 contiguous bytes)
                const float4* tile = reinterpret_cast<const float4*>(smem + st * kTileBytes);
                const int r0 = cwarp * 8 + 2 * (lane >> 3), sl = lane & 7;
                float4 s[2][4];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                    for (int i = 0; i < 4; ++i) s[rr][i] = tile[(r0 + rr) * 32 + sl + 8 * i];
                __syncwarp();
                if (lane == 0 && !broken) mbar_arrive(&empty[st]);  // this warp is done reading the stage
                // after the reduction lane l holds row r0 + ((l >> 2) & 1), S.k if bit 1 of l is clear, else S.q
                const int irow = half * 64 + r0 + ((lane >> 2) & 1);
#pragma unroll 1
                for (int j = 0; j < nt; ++j) {
                    {
                        const float alpha = s_gate[2 * (j * G + hh)], beta = s_gate[2 * (j * G + hh) + 1];
                        const float4* q4 = reinterpret_cast<const float4*>(s_q + j * 128) + sl;
                        const float4* k4 = reinterpret_cast<const float4*>(s_k + j * 128) + sl;
                        float4 kf[4], qf[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            kf[i] = k4[8 * i];
                            qf[i] = q4[8 * i];
                        }
                        float v[4] = {dot16(s[0], kf), dot16(s[0], qf), dot16(s[1], kf), dot16(s[1], qf)};
                        const float tot = group8_transpose_sum4(v, lane);
                        const float u_k = beta * fmaf(-alpha, tot, s_v[(j * G + hh) * 128 + irow]);  // lanes with bit 1 clear
                        const float u0 = __shfl_sync(0xffffffffu, u_k, lane & ~7);        // row r0
                        const float u1 = __shfl_sync(0xffffffffu, u_k, (lane & ~7) | 4);  // row r0 + 1
                        if ((lane & 3) == 2)
                            s_o[(j * G + hh) * 128 + irow] = fmaf((lane & 4) ? u1 : u0, s_kq[j], alpha * tot);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            s[0][i] = decay_add(s[0][i], alpha, u0, kf[i]);
                            s[1][i] = decay_add(s[1][i], alpha, u1, kf[i]);
                        }
                    }
                }
                float4* gdst = reinterpret_cast<float4*>(unit_ptr(u));
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                    for (int i = 0; i < 4; ++i) __stcs(gdst + (r0 + rr) * 32 + sl + 8 * i, s[rr][i]);
            }
        }

        // ---- gated RMSNorm of the G heads' 128 outputs of every token
        named_barrier_sync(gbar, kComputeThreads);
#pragma unroll 1
        for (int j = 0; j < nt; ++j) {
            {
                for (int hh = 0; hh < G; ++hh) {
                    const float o = (ctid < 128) ? s_o[(j * G + hh) * 128 + ctid] : 0.f;
                    const float ss = warp_sum(o * o);
                    if (lane == 0) s_red[j * nred + 8 + hh * 8 + cwarp] = ss;
                }
            }
        }
        named_barrier_sync(gbar, kComputeThreads);
        if (ctid < 128) {
            const uint16_t* az = reinterpret_cast<const uint16_t*>(ax + pl.aux_z);
#pragma unroll 1
            for (int j = 0; j < nt; ++j) {
                {
                    for (int hh = 0; hh < G; ++hh) {
                        const float* r4 = s_red + j * nred + 8 + hh * 8;
                        const float ms = (r4[0] + r4[1] + r4[2] + r4[3]) * (1.0f / 128.0f);
                        const int head = kap * Gfull + hoff + hh;
                        const float zv = bf16_bits_to_float(az[(j * G + hh) * 128 + ctid]);
                        const float y = s_o[(j * G + hh) * 128 + ctid] * rsqrtf(ms + kEps) * w_n * silu_f(zv);
                        p.out[(((size_t)row * nt + j) * p.Vh + head) * 128 + ctid] = float_to_bf16_bits(y);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0 && !broken) mbar_arrive(&auxempty[m & 1]);  // this warp is done with the item's inputs
    }
    // Split group: the peers signal rank 0's q/k-history barrier in rank 0's shared memory.  If
    // rank 0 gave up waiting for them, it still holds until they have signalled (fixed bound),
    // so no remote arrive reaches a CTA that has exited.
    if (SPLIT && tid == 0 && nmine > 0) {
        int row, kap, hoff;
        item(blockIdx.x, row, kap, hoff);
        if (hoff == 0) mbar_wait(qkfree, 0);
    }
}

}  // namespace gdn
