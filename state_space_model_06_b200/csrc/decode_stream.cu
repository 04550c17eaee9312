// decode_stream.cu -- MIMO decode step (N = 64, P = 64, rank 2 or 4; the output gate, the
// BC map and the lightweight expansion fused) as a persistent streaming kernel.
//
// Mamba-3 paper summary, "Multi-Input, Multi-Output Formulation": at decode time each
// head's N x P fp32 state is read and written once per token, so the step is bound by
// HBM.  With one CTA per head, each CTA's 16 KB state is loaded into registers, updated
// and stored, and an SM only has the loads of its resident CTAs in flight while they
// compute: a copy-only version of that shape stops at about two thirds of HBM.
//
// Here each warp owns a stream of heads (bh = global warp, + number of warps, ...): the
// 16 KB state arrives in shared memory by one bulk copy into the warp's slot, the per-head
// factors are built by the warp itself (one lane per state pair) while the copy flies,
// and the warp needs no CTA-wide barrier.  For N = 64 eight warps per SM, two on each
// sub-partition: while one waits for its copy the other updates its head.  For N = 128
// (SISO) a head's 32 KB state is split into two 16 KB halves of its rows, each updated by
// one warp of a stream (four warps per SM, two slots each); the readout's sum over N then
// meets in shared memory (see the exchange below).  The update is the one of the per-head
// kernels:
//   h' = R(phi)(alpha h) + [beta R(phi) Bp | gamma B] [xp | x]^T,
//   Y  = h'^T C + D x  (times SiLU(z) with the output gate),
// on packed fp32 pairs, with the new state written from registers straight to HBM.
// Lane (j, half) holds column chunk j (4 columns) and the state pairs half*16 .. +15.
#include "m3_internal.h"
#include "sm100.cuh"

namespace m3 {

using namespace sm100;

namespace {

// warps per CTA (one CTA per SM) and state slots per warp (heads in flight), whole heads
// (HV = 1) and half-heads (HV = 2).  Measured per batch-256 step on B200: whole rank-4 heads
// 8 x 1 102.6 us (6 x 1 117, 4 x 2 127, 5 x 2 133); SISO half-heads 4 x 2 172.9 us (8 x 1
// 189.3, 6 x 2 188.6, 4 x 3 182.0).  The heads are dealt to the warps statically, so the four
// SM sub-partitions must carry equal numbers of warps.
constexpr int kSW1 = 8, kSlots1 = 1;
constexpr int kSW2 = 4, kSlots2 = 2;
constexpr int kNP = 32;                          // state pairs (N = 64)
constexpr int kPc = 64;                          // columns (P = 64)
constexpr int kStateBytes = 2 * kNP * kPc * 4;   // 16 KB per head

constexpr int kEx = 4;                           // readout exchange slots per stream (HV = 2)

// HV: warps per head.  1: a warp updates a whole head (N = 64).  2 (N = 128): the two
// warps of a stream update one half of the head's state rows each, and the second to
// finish adds the other's readout partial.
template <int R, int HV>
struct SCfg {
    static constexpr int SW = HV == 1 ? kSW1 : kSW2;
    static constexpr int SLOTS = HV == 1 ? kSlots1 : kSlots2;
    static constexpr int FAC_F4 = kNP * (2 + 3 * R);   // rot [2], U [2R], C [R] per pair
    static constexpr int WARP_BYTES = SLOTS * kStateBytes + FAC_F4 * 16;
    static constexpr int STREAMS = SW / HV;            // head streams per CTA
    static constexpr int OFF_EX = SW * WARP_BYTES + SW * SLOTS * 8;   // exchange area
    static constexpr int EX_FLOATS = HV == 2 ? STREAMS * kEx * 2 * R * kPc : 0;
    static constexpr int EX_BYTES = HV == 2 ? EX_FLOATS * 4 + STREAMS * kEx * 4 : 0;
    static constexpr int SMEM = OFF_EX + EX_BYTES + 128;   // + alignment
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(OFF_EX % 16 == 0, "exchange alignment");
};

__device__ __forceinline__ float2 lo2(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4& v) { return make_float2(v.z, v.w); }

// four consecutive io values as floats
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
}
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
// the two values of a state pair (rows 2i, 2i+1) of one rank column
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(bf16lo(u), bf16hi(u));
}
__device__ __forceinline__ float2 load2(const float* p) { return *reinterpret_cast<const float2*>(p); }

// v * w rounded to the io dtype, four channels (the MIMO lightweight expansion)
template <typename IO>
__device__ __forceinline__ float4 expand4(float4 v, float4 w) {
    return make_float4(expand_io<IO>(v.x, w.x), expand_io<IO>(v.y, w.y), expand_io<IO>(v.z, w.z),
                       expand_io<IO>(v.w, w.w));
}

// The small per-head inputs, fetched one head ahead into registers.
// XE: x (and z with z_expand) hold one value per head channel, [b][H][P], and rank column r
// is that value times the head's weight w[r][p], rounded to the io dtype ("Multi-Input,
// Multi-Output (MIMO) Formulation", MIMO Parameterization Choices).
// HV = 2 (half-heads) with the BC map: the lane also holds the squares of the same pair of
// the other half of N, so that each warp forms the column RMS over all N on its own.
template <typename IO, int R, bool BCM, bool XE, int HV = 1>
struct Small {
    float dt, A, lam, th, D;
    float2 bq[R], bp[R], cc[R];   // this lane's pair (rows 2 lane, 2 lane + 1) of B, B_prev, C
    float2 biasB, biasC;          // the head's BC biases of this lane's pair (BC map)
    float oq[R], op[R], oc[R];    // HV = 2, BC map: squares of the other half's pair
    float4 x[R], xp[R], z[R];     // this lane's column chunk of x, x_prev, z (rank columns)
    // pb: the first state pair of this warp's rows
    __device__ void load(const DecodeArgs& a, int bh, int lane, int pb) {
        const int H = a.H, G = a.G, N = a.N, P = a.P;
        const int b = bh / H, h = bh - b * H, g = h / (H / G);
        const int j = lane & 15, pr = pb + lane;
        dt = a.dt[bh];
        A = a.A[bh];
        lam = a.lam[bh];
        D = a.D ? a.D[h] : 0.f;
        th = a.theta[((size_t)b * G + g) * (N / 2) + pr];
        const size_t gofs = ((size_t)b * G + g) * R * N + 2 * pr;
        const IO* Bg = static_cast<const IO*>(a.B) + gofs;
        const IO* Bpg = static_cast<const IO*>(a.B_prev) + gofs;
        const IO* Cg = static_cast<const IO*>(a.C) + gofs;
        if constexpr (BCM) {
            biasB = a.B_bias ? load2(a.B_bias + (size_t)h * N + 2 * pr) : make_float2(0.f, 0.f);
            biasC = a.C_bias ? load2(a.C_bias + (size_t)h * N + 2 * pr) : make_float2(0.f, 0.f);
        }
        const size_t xofs = (size_t)bh * R * P + 4 * j;
        const IO* xp0 = static_cast<const IO*>(a.x_prev) + xofs;
        const bool xe = XE && a.x_expand, ze = XE && a.z_expand;
        float4 x1 = make_float4(0.f, 0.f, 0.f, 0.f), z1 = x1;
        if (xe) x1 = load4(static_cast<const IO*>(a.x) + (size_t)bh * P + 4 * j);
        if (ze) z1 = load4(static_cast<const IO*>(a.z) + (size_t)bh * P + 4 * j);
        const float* wx = xe ? a.x_expand + ((size_t)h * R) * P + 4 * j : nullptr;
        const float* wz = ze ? a.z_expand + ((size_t)h * R) * P + 4 * j : nullptr;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            bq[r] = load2(Bg + r * N);
            bp[r] = load2(Bpg + r * N);
            cc[r] = load2(Cg + r * N);
            if constexpr (BCM && HV == 2) {
                const int other = 2 * (kNP - 2 * pb);   // element offset of the partner pair
                const float2 q2 = load2(Bg + r * N + other), p2 = load2(Bpg + r * N + other),
                             c2 = load2(Cg + r * N + other);
                oq[r] = q2.x * q2.x + q2.y * q2.y;
                op[r] = p2.x * p2.x + p2.y * p2.y;
                oc[r] = c2.x * c2.x + c2.y * c2.y;
            }
            x[r] = xe ? expand4<IO>(x1, load4(wx + r * P))
                      : load4(static_cast<const IO*>(a.x) + xofs + r * P);
            xp[r] = load4(xp0 + r * P);
            if (ze)
                z[r] = expand4<IO>(z1, load4(wz + r * P));
            else
                z[r] = a.z ? load4(static_cast<const IO*>(a.z) + xofs + r * P)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <typename IO, int R, bool BCM, bool XE, int HV>
__global__ void __launch_bounds__((HV == 1 ? kSW1 : kSW2) * 32, 1)
    decode_stream_kernel(DecodeArgs a, int nbh) {
    using C = SCfg<R, HV>;
    static_assert(HV == 1 || (HV == 2 && !XE), "half-heads run SISO without the expansion");
    constexpr int R2 = 2 * R;
    extern __shared__ __align__(128) uint8_t sm_raw[];
    uint8_t* smb = sm_raw + ((128u - (smem_u32(sm_raw) & 127u)) & 127u);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = lane & 15, half = lane >> 4;
    uint8_t* wb = smb + w * C::WARP_BYTES;
    const float* slot0 = reinterpret_cast<const float*>(wb);
    constexpr int kSlots = C::SLOTS;
    float4* rot4 = reinterpret_cast<float4*>(wb + kSlots * kStateBytes);   // [32][2]
    float4* U4 = rot4 + kNP * 2;                                       // [32][2R]
    float4* C4 = U4 + kNP * R2;                                        // [32][R]
    uint64_t* bar = reinterpret_cast<uint64_t*>(smb + C::SW * C::WARP_BYTES) + kSlots * w;
    if (lane == 0) {
        for (int s = 0; s < kSlots; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    if constexpr (HV == 2) {   // the exchange counters start at 0 before any warp uses them
        unsigned* c0 = reinterpret_cast<unsigned*>(reinterpret_cast<float*>(smb + C::OFF_EX) +
                                                   C::EX_FLOATS);
        for (int k = threadIdx.x; k < C::STREAMS * kEx; k += blockDim.x) c0[k] = 0u;
        __syncthreads();
    }

    // head stream sw of the CTA; with HV = 2 warp w updates the state rows of half hf
    const int sw = w % C::STREAMS, hf = w / C::STREAMS;
    const int gw = blockIdx.x * C::STREAMS + sw, NW = gridDim.x * C::STREAMS;
    const int nmine = gw < nbh ? (nbh - gw + NW - 1) / NW : 0;
    constexpr size_t kHeadFloats = (size_t)HV * 2 * kNP * kPc;
    const size_t hoff = (size_t)hf * 2 * kNP * kPc;   // this warp's rows within the head
    auto issue = [&](int i) {   // lane 0: the state of this warp's i-th head into its slot
        const int s = i % kSlots;
        mbar_arrive_expect_tx(&bar[s], kStateBytes);
        bulk_load(wb + s * kStateBytes, a.h + (size_t)(gw + i * NW) * kHeadFloats + hoff,
                  kStateBytes, &bar[s]);
    };
    if (lane == 0)
        for (int i = 0; i < kSlots && i < nmine; ++i) issue(i);
    Small<IO, R, BCM, XE, HV> nx;
    if (nmine > 0) nx.load(a, gw, lane, hf * kNP);
    const bool angle = (a.flags & M3_FLAG_THETA_IS_ANGLE) != 0;
    int issued = nmine < kSlots ? nmine : kSlots;   // copies issued
    bool ok = true;

    for (int i = 0; i < nmine && ok; ++i) {
        const int bh = gw + i * NW;
        Small<IO, R, BCM, XE, HV> cur = nx;
        if constexpr (BCM) {
            // BC map ("Technical Approach", BCNorm and BC biases): each rank column of B,
            // B_prev and C scaled to unit RMS over N (when bc_eps > 0; the lanes hold the
            // column's N values as pairs), plus the head's channel bias
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float sq = 1.f, sp = 1.f, sc = 1.f;
                if (a.bc_eps > 0.f) {
                    const float invn = 1.f / (float)a.N;
                    float eq = 0.f, ep = 0.f, ec = 0.f;
                    if constexpr (HV == 2) {
                        eq = cur.oq[r];
                        ep = cur.op[r];
                        ec = cur.oc[r];
                    }
                    sq = rsqrtf(warp_sum(cur.bq[r].x * cur.bq[r].x + cur.bq[r].y * cur.bq[r].y + eq) * invn + a.bc_eps);
                    sp = rsqrtf(warp_sum(cur.bp[r].x * cur.bp[r].x + cur.bp[r].y * cur.bp[r].y + ep) * invn + a.bc_eps);
                    sc = rsqrtf(warp_sum(cur.cc[r].x * cur.cc[r].x + cur.cc[r].y * cur.cc[r].y + ec) * invn + a.bc_eps);
                }
                cur.bq[r] = make_float2(fmaf(cur.bq[r].x, sq, cur.biasB.x), fmaf(cur.bq[r].y, sq, cur.biasB.y));
                cur.bp[r] = make_float2(fmaf(cur.bp[r].x, sp, cur.biasB.x), fmaf(cur.bp[r].y, sp, cur.biasB.y));
                cur.cc[r] = make_float2(fmaf(cur.cc[r].x, sc, cur.biasC.x), fmaf(cur.cc[r].y, sc, cur.biasC.y));
            }
        }
        // ---- this head's factors: lane = state pair
        {
            const float alpha = expf(cur.dt * cur.A);
            const float beta = (1.f - cur.lam) * cur.dt * alpha;
            const float gamma = cur.lam * cur.dt;
            float sn, cs;
            sincosf(angle ? cur.th : cur.dt * cur.th, &sn, &cs);
            const float ac = alpha * cs, as = alpha * sn;
            rot4[2 * lane] = make_float4(ac, ac, as, as);
            rot4[2 * lane + 1] = make_float4(-as, -as, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float p0 = cur.bp[r].x, p1 = cur.bp[r].y;
                const float ub0 = beta * (cs * p0 - sn * p1), ub1 = beta * (sn * p0 + cs * p1);
                const float ug0 = gamma * cur.bq[r].x, ug1 = gamma * cur.bq[r].y;
                U4[lane * R2 + r] = make_float4(ub0, ub0, ub1, ub1);
                U4[lane * R2 + R + r] = make_float4(ug0, ug0, ug1, ug1);
                C4[lane * R + r] = make_float4(cur.cc[r].x, cur.cc[r].x, cur.cc[r].y, cur.cc[r].y);
            }
        }
        __syncwarp();
        // the next head's small inputs fly while this one is updated
        if (i + 1 < nmine) nx.load(a, bh + NW, lane, hf * kNP);

        // ---- wait for this head's state (bounded)
        const int s = i % kSlots;
        const uint32_t par = (i / kSlots) & 1;
        {
            const uint64_t t0 = globaltimer();
            bool got = mbar_try_wait(&bar[s], par);
            while (!got && globaltimer() - t0 < 2000000000ull)
                got = mbar_try_wait_hint(&bar[s], par, 20000u);
            ok = __all_sync(0xffffffffu, got);
        }
        float2 ya[R], yb[R];
#pragma unroll
        for (int r = 0; r < R; ++r) ya[r] = yb[r] = make_float2(0.f, 0.f);
        if (ok) {
            const float* st = slot0 + s * (kStateBytes / 4);
            float4* hrow = reinterpret_cast<float4*>(a.h + (size_t)bh * kHeadFloats + hoff);
#pragma unroll 2
            for (int kk = 0; kk < kNP / 2; ++kk) {
                const int ip = half * (kNP / 2) + kk;
                const float4 h0 = *reinterpret_cast<const float4*>(st + (2 * ip) * kPc + 4 * j);
                const float4 h1 = *reinterpret_cast<const float4*>(st + (2 * ip + 1) * kPc + 4 * j);
                const float4 rc = rot4[2 * ip], rn = rot4[2 * ip + 1];
                // row 2i: ac h0 - as h1;  row 2i+1: as h0 + ac h1
                float2 n0a = __ffma2_rn(lo2(rc), lo2(h0), __fmul2_rn(lo2(rn), lo2(h1)));
                float2 n0b = __ffma2_rn(lo2(rc), hi2(h0), __fmul2_rn(lo2(rn), hi2(h1)));
                float2 n1a = __ffma2_rn(hi2(rc), lo2(h0), __fmul2_rn(lo2(rc), lo2(h1)));
                float2 n1b = __ffma2_rn(hi2(rc), hi2(h0), __fmul2_rn(lo2(rc), hi2(h1)));
#pragma unroll
                for (int q = 0; q < R2; ++q) {
                    const float4 u = U4[ip * R2 + q];
                    const float4 v = q < R ? cur.xp[q] : cur.x[q - R];
                    n0a = __ffma2_rn(lo2(u), lo2(v), n0a);
                    n0b = __ffma2_rn(lo2(u), hi2(v), n0b);
                    n1a = __ffma2_rn(hi2(u), lo2(v), n1a);
                    n1b = __ffma2_rn(hi2(u), hi2(v), n1b);
                }
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float4 c = C4[ip * R + r];
                    ya[r] = __ffma2_rn(n0a, lo2(c), __ffma2_rn(n1a, hi2(c), ya[r]));
                    yb[r] = __ffma2_rn(n0b, lo2(c), __ffma2_rn(n1b, hi2(c), yb[r]));
                }
                __stcs(hrow + (size_t)(2 * ip) * (kPc / 4) + j, make_float4(n0a.x, n0a.y, n0b.x, n0b.y));
                __stcs(hrow + (size_t)(2 * ip + 1) * (kPc / 4) + j,
                       make_float4(n1a.x, n1a.y, n1b.x, n1b.y));
            }
        }
        // ---- readout: the two halves' partial sums over the state rows
#pragma unroll
        for (int r = 0; r < R; ++r) {
            ya[r].x += __shfl_xor_sync(0xffffffffu, ya[r].x, 16);
            ya[r].y += __shfl_xor_sync(0xffffffffu, ya[r].y, 16);
            yb[r].x += __shfl_xor_sync(0xffffffffu, yb[r].x, 16);
            yb[r].y += __shfl_xor_sync(0xffffffffu, yb[r].y, 16);
        }
        bool writer = true;   // this warp writes y and x_prev
        if constexpr (HV == 2) {
            // The two warps of the stream meet through exchange slot i % kEx: each writes
            // its partial readout there and arrives on the slot's counter; the second to
            // arrive adds the other's partial and writes the head's outputs, then arrives
            // once more to free the slot.  Use u = i / kEx of a slot spans counter values
            // 3u .. 3u + 3; a warp more than kEx heads ahead of its partner waits (bounded)
            // until the slot's previous use is over.
            float* exb = reinterpret_cast<float*>(smb + C::OFF_EX);
            unsigned* cnt = reinterpret_cast<unsigned*>(exb + C::EX_FLOATS) + sw * kEx;
            const int es = i % kEx;
            const unsigned base = 3u * (unsigned)(i / kEx);
            bool fr = true;
            if (lane == 0) {
                const uint64_t t0 = globaltimer();
                while (*reinterpret_cast<volatile unsigned*>(&cnt[es]) < base &&
                       globaltimer() - t0 < 2000000000ull) {
                }
                fr = *reinterpret_cast<volatile unsigned*>(&cnt[es]) >= base;
            }
            fr = __shfl_sync(0xffffffffu, fr ? 1 : 0, 0) != 0;
            if (!fr) ok = false;
            float* mine = exb + ((size_t)(sw * kEx + es) * 2 + hf) * R * kPc;
            const float* other = exb + ((size_t)(sw * kEx + es) * 2 + (hf ^ 1)) * R * kPc;
            if (half == 0) {
#pragma unroll
                for (int r = 0; r < R; ++r)
                    *reinterpret_cast<float4*>(mine + r * kPc + 4 * j) =
                        make_float4(ya[r].x, ya[r].y, yb[r].x, yb[r].y);
            }
            __syncwarp();
            unsigned old = 0;
            if (lane == 0) {
                __threadfence_block();
                old = atomicAdd(&cnt[es], 1u);
                __threadfence_block();
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            writer = old == base + 1;
            if (writer && half == 0) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const float4 o = *reinterpret_cast<const float4*>(other + r * kPc + 4 * j);
                    ya[r].x += o.x; ya[r].y += o.y; yb[r].x += o.z; yb[r].y += o.w;
                }
            }
        }
        if (writer && half == 0) {
            IO* y = static_cast<IO*>(a.y) + (size_t)bh * R * kPc + 4 * j;
            IO* xpo = static_cast<IO*>(a.x_prev) + (size_t)bh * R * kPc + 4 * j;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float4 v = make_float4(ya[r].x, ya[r].y, yb[r].x, yb[r].y);
                if (!ok) v = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                         __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
                v.x = fmaf(cur.D, cur.x[r].x, v.x);
                v.y = fmaf(cur.D, cur.x[r].y, v.y);
                v.z = fmaf(cur.D, cur.x[r].z, v.z);
                v.w = fmaf(cur.D, cur.x[r].w, v.w);
                if (a.z) {
                    v.x = gate_silu(v.x, cur.z[r].x);
                    v.y = gate_silu(v.y, cur.z[r].y);
                    v.z = gate_silu(v.z, cur.z[r].z);
                    v.w = gate_silu(v.w, cur.z[r].w);
                }
                store4(y + r * kPc, v);
                store4(xpo + r * kPc, cur.x[r]);   // x_prev <- x (exact in the io dtype)
            }
        }
        if constexpr (HV == 2) {
            if (writer) {   // the other warp's partial is read: free the exchange slot
                __syncwarp();
                if (lane == 0) {
                    __threadfence_block();
                    atomicAdd(reinterpret_cast<unsigned*>(reinterpret_cast<float*>(smb + C::OFF_EX) +
                                                          C::EX_FLOATS) + sw * kEx + i % kEx,
                              1u);
                }
            }
        }
        // the slot is free once every lane has read it: the copy of head i + kSlots goes there
        __syncwarp();
        fence_proxy_async_smem();
        if (ok && lane == 0 && i + kSlots < nmine) {
            issue(i + kSlots);
            ++issued;
        }
    }
    if (!ok && lane == 0) {
        // a copy did not land in time (this head's y is NaN): let the copies issued into
        // each slot land (bounded) before the CTA's shared memory is released
        for (int s = 0; s < kSlots; ++s) {
            const int n = (issued - s + kSlots - 1) / kSlots;   // copies issued into slot s
            if (n == 0) continue;
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&bar[s], (n - 1) & 1) && globaltimer() - t0 < 10000000ull) {
            }
        }
    }
}

int num_sms() {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            sms[dev] = n;
    }
    return sms[dev] ? sms[dev] : 148;
}

template <typename IO, int R, bool BCM, bool XE, int HV = 1>
cudaError_t launch_stream_t(const DecodeArgs& a, int batch, cudaStream_t s) {
    using C = SCfg<R, HV>;
    cudaError_t e = cudaFuncSetAttribute(decode_stream_kernel<IO, R, BCM, XE, HV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const int nbh = batch * a.H;
    int grid = num_sms();
    const int need = (nbh + C::STREAMS - 1) / C::STREAMS;
    if (grid > need) grid = need;
    decode_stream_kernel<IO, R, BCM, XE, HV><<<grid, C::SW * 32, C::SMEM, s>>>(a, nbh);
    return cudaGetLastError();
}

template <typename IO, bool BCM, bool XE>
cudaError_t launch_stream_r(const DecodeArgs& a, int batch, int R, cudaStream_t s) {
    return R == 2 ? launch_stream_t<IO, 2, BCM, XE>(a, batch, s)
                  : launch_stream_t<IO, 4, BCM, XE>(a, batch, s);
}

template <typename IO>
cudaError_t launch_stream_io(const DecodeArgs& a, int batch, int R, cudaStream_t s) {
    const bool bcm = a.B_bias || a.C_bias || a.bc_eps > 0.f;
    const bool xe = a.x_expand || a.z_expand;
    if (bcm) return xe ? launch_stream_r<IO, true, true>(a, batch, R, s)
                       : launch_stream_r<IO, true, false>(a, batch, R, s);
    return xe ? launch_stream_r<IO, false, true>(a, batch, R, s)
              : launch_stream_r<IO, false, false>(a, batch, R, s);
}

}  // namespace

// MIMO N = 64 (rank 2, 4; every fused part), and SISO N = 128 as half-heads (plain, with
// the output gate and with the BC map; each half-head warp forms the column RMS over all N)
bool decode_stream_ok(const DecodeArgs& a, int R) {
    if (a.P != kPc) return false;
    if (a.N == 2 * kNP) return R == 2 || R == 4;
    return a.N == 4 * kNP && R == 1 && !a.x_expand && !a.z_expand;
}

// The BC map and the lightweight expansion are compile-time variants, so the plain
// instantiations hold none of their code.
cudaError_t launch_decode_stream(const DecodeArgs& a, int batch, int R, int io_dtype,
                                 cudaStream_t s) {
    if (a.N == 4 * kNP) {
        const bool bcm = a.B_bias || a.C_bias || a.bc_eps > 0.f;
        if (bcm)
            return io_dtype == M3_BF16 ? launch_stream_t<__nv_bfloat16, 1, true, false, 2>(a, batch, s)
                                       : launch_stream_t<float, 1, true, false, 2>(a, batch, s);
        return io_dtype == M3_BF16 ? launch_stream_t<__nv_bfloat16, 1, false, false, 2>(a, batch, s)
                                   : launch_stream_t<float, 1, false, false, 2>(a, batch, s);
    }
    return io_dtype == M3_BF16 ? launch_stream_io<__nv_bfloat16>(a, batch, R, s)
                               : launch_stream_io<float>(a, batch, R, s);
}

}  // namespace m3
