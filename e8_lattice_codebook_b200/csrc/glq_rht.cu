// glq_rht.cu -- the two Randomized Hadamard Transform stages of the GLQ
// linear layer (glq 0.5.1 PyPI page, "How it works" 2: random sign flips
// followed by a fast Walsh-Hadamard transform; "Bit widths": block-diagonal
// transform over the binary decomposition of a size that is not a power of
// two; GLQ v0.3.2 / v0.3.3 release notes: input_rht / output_rht, and a
// separate path above 16384).
//
// Design (B200): a row is cut into parts of at most 4096 values; the parts
// of one row form one thread-block cluster (<= 8 CTAs).  A block of the
// decomposition larger than 4096 is split into C = K/4096 consecutive
// parts, using H_K = (H_C (x) I_{K/C}) (I_C (x) H_{K/C}):
//   1. each part transforms its own 4096 values in shared memory (radix-16
//      rounds in registers over a padded, conflict-free layout);
//   2. after a cluster barrier, part q combines position i of all C parts
//      (distributed shared memory loads, an in-register H_C) for its 1/C of
//      the positions and writes all C outputs of those positions.
// Smaller blocks are packed whole into parts and finish after step 1.
// The input side then finds the row's max |xr| (cluster reduction), picks a
// power-of-two scale and writes the activations as 16-bit integers (split
// into high and low bytes for the integer MMA of the GEMV) and as fp16,
// with the exact integer sum of the row.
#include <cooperative_groups.h>

#include <cmath>

#include "glq_kernels.cuh"

namespace cg = cooperative_groups;

namespace glq {

namespace {

constexpr int SEG = GLQ_RHT_SEG;          // values per part (4096)
constexpr int THREADS = GLQ_RHT_THREADS;  // threads per part (1024)
constexpr int VPT = SEG / THREADS;        // values per thread (4), consecutive

// Shared-memory index of row-local position i.  No padding: every access
// pattern below has consecutive lanes on consecutive positions, and the
// float4 accesses at 4t need 16-byte alignment.
__device__ __forceinline__ int padi(int i) { return i; }

__device__ __forceinline__ bool sign_neg(const uint32_t *bits, int k) {
    return (bits[k >> 5] >> (k & 31)) & 1u;
}

__device__ __forceinline__ int ilog2(int v) { return 31 - __clz(v); }

// The piece of the part holding local position L (pieces are packed in
// descending, power-of-two sizes, so each starts at a multiple of its size).
__device__ __forceinline__ int piece_of(const RhtPlan &plan, int part, int L, int &lo) {
    const int p0 = plan.first_piece[part], p1 = plan.first_piece[part + 1];
    int pc = p0, base = 0;
    while (pc + 1 < p1 && L >= base + plan.piece[pc].len) {
        base += plan.piece[pc].len;
        ++pc;
    }
    lo = base;
    return pc;
}

struct Outputs {
    float v[VPT];
    int idx[VPT];  // position within the row, -1 if unused
};

// Local unnormalised transform of a part: thread t owns local positions
// 4t..4t+3 (values v[0..3]) inside a piece of log2-size lk.  Bits 0-1 in
// registers, bits 2-6 across the lanes of a warp, bits 7-11 through shared
// memory in radix-4 rounds.  `buf` holds SEG floats.  All threads
// call it; it ends synchronised with the result back in v.
__device__ __forceinline__ void local_fwht(float v[4], int lk, float *buf, const RhtPlan &plan, int part) {
    // bits 0, 1
    if (lk > 0) {
        float a = v[0], b = v[1], c = v[2], d = v[3];
        v[0] = a + b; v[1] = a - b; v[2] = c + d; v[3] = c - d;
    }
    if (lk > 1) {
        float a = v[0], b = v[1], c = v[2], d = v[3];
        v[0] = a + c; v[1] = b + d; v[2] = a - c; v[3] = b - d;
    }
    // bits 2..6: partner lane = lane ^ (1 << (bit - 2))
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int bit = 2; bit < 7; ++bit) {
        const int m = 1 << (bit - 2);
        const bool upper = lane & m;
        const bool active = bit < lk;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
            if (active) v[i] = upper ? o - v[i] : v[i] + o;
        }
    }
    // bits 7..11 through shared memory
    const int t = threadIdx.x;
    const int lk_max = ilog2(plan.piece[plan.first_piece[part]].len);  // largest piece first
    if (lk_max <= 7) return;  // no piece extends past bit 6
    *reinterpret_cast<float4 *>(&buf[padi(4 * t)]) = make_float4(v[0], v[1], v[2], v[3]);
    __syncthreads();
    for (int b0 = 7; b0 < lk_max;) {
        // A butterfly on (p, p + 2^bit) applies iff bit < log2 of p's piece
        // (pieces are aligned to their power-of-two sizes, so the test is
        // symmetric).
        const int s = 1 << b0;
        const int lowmask = s - 1;
        if (lk_max - b0 >= 2) {
            // radix 4 over bits b0, b0+1: group t = positions base + {0,s,2s,3s}
            const int base = ((t & ~lowmask) << 2) | (t & lowmask);
            int lo;
            const int lkA = ilog2(plan.piece[piece_of(plan, part, base, lo)].len);
            const int lkB = ilog2(plan.piece[piece_of(plan, part, base + 2 * s, lo)].len);
            float a = buf[padi(base)], b = buf[padi(base + s)];
            float c = buf[padi(base + 2 * s)], d = buf[padi(base + 3 * s)];
            if (b0 < lkA) {
                const float x = a + b, y = a - b;
                a = x;
                b = y;
            }
            if (b0 < lkB) {
                const float x = c + d, y = c - d;
                c = x;
                d = y;
            }
            if (b0 + 1 < lkA) {
                const float x = a + c, y = a - c, u = b + d, w = b - d;
                a = x;
                c = y;
                b = u;
                d = w;
            }
            buf[padi(base)] = a;
            buf[padi(base + s)] = b;
            buf[padi(base + 2 * s)] = c;
            buf[padi(base + 3 * s)] = d;
            b0 += 2;
        } else {
            // radix 2 over bit b0: pairs q = t and t + THREADS
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int q = t + h * THREADS;
                const int base = ((q & ~lowmask) << 1) | (q & lowmask);
                int lo;
                const int lkA = ilog2(plan.piece[piece_of(plan, part, base, lo)].len);
                if (b0 < lkA) {
                    const float a = buf[padi(base)], b = buf[padi(base + s)];
                    buf[padi(base)] = a + b;
                    buf[padi(base + s)] = a - b;
                }
            }
            b0 += 1;
        }
        __syncthreads();
    }
    const float4 r = *reinterpret_cast<const float4 *>(&buf[padi(4 * t)]);
    v[0] = r.x; v[1] = r.y; v[2] = r.z; v[3] = r.w;
}

// Cross stage of a block split over C parts: this part owns positions
// [q SEG/C, (q+1) SEG/C) of every part and produces the C outputs of each
// (one in-register H_C over values read from the C parts' shared memory).
// C = 2: two positions per thread; C = 4: one; C = 8: half of one.
template <int C>
__device__ __forceinline__ void cross_stage(const RhtPiece &first, float *buf, Outputs &o,
                                            cg::cluster_group &cluster) {
    constexpr int SPAN = SEG / C;
    constexpr int NPOS = SPAN >= THREADS ? SPAN / THREADS : 1;  // positions per thread
    constexpr int TPP = SPAN >= THREADS ? 1 : THREADS / SPAN;   // threads per position
    constexpr int JN = C / TPP;                                // outputs per position per thread
    static_assert(NPOS * JN == VPT, "every thread produces VPT outputs");
    const int t = threadIdx.x;
    const float *peer[C];
#pragma unroll
    for (int j = 0; j < C; ++j) peer[j] = cluster.map_shared_rank(buf, first.rank0 + j);
    const int blk_off = first.off - first.q * SEG;
    const int half = TPP == 1 ? 0 : t / SPAN;  // which JN outputs of the position
#pragma unroll
    for (int pi = 0; pi < NPOS; ++pi) {
        const int pos = TPP == 1 ? t + pi * THREADS : t % SPAN;
        const int i = first.q * SPAN + pos;
        float w[C];
#pragma unroll
        for (int j = 0; j < C; ++j) w[j] = peer[j][padi(i)];
#pragma unroll
        for (int h = 1; h < C; h <<= 1)
#pragma unroll
            for (int k = 0; k < C; ++k)
                if ((k & h) == 0) {
                    const float a = w[k], b = w[k + h];
                    w[k] = a + b;
                    w[k + h] = a - b;
                }
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) {
            const int j = half * JN + jj;
            const float val = TPP == 1 ? w[jj] : (half ? w[(JN + jj) % C] : w[jj]);
            o.v[pi * JN + jj] = val * first.norm;
            o.idx[pi * JN + jj] = blk_off + j * SEG + i;
        }
    }
}

// Transform of one part: its 4 values per thread (already loaded, signs
// applied), local transform, cross stage of a block split over C parts,
// outputs (normalised) with their row positions.  All threads of all CTAs of
// the cluster call it (it holds cluster barriers).
__device__ __forceinline__ void part_transform(const RhtPlan &plan, int part, float *buf, float v[4],
                                               int part_len, Outputs &o, cg::cluster_group &cluster) {
    const int L = 4 * threadIdx.x;
    int lo = 0;
    const int pc = piece_of(plan, part, L < part_len ? L : 0, lo);
    const RhtPiece P = plan.piece[pc];
    local_fwht(v, ilog2(P.len), buf, plan, part);
#pragma unroll
    for (int i = 0; i < VPT; ++i) o.idx[i] = -1;

    const RhtPiece first = plan.piece[plan.first_piece[part]];
    // a part of a split block publishes its local result; every part of the
    // cluster then takes the same barrier (cluster barriers must match)
    if (first.C > 1) *reinterpret_cast<float4 *>(&buf[padi(L)]) = make_float4(v[0], v[1], v[2], v[3]);
    if (plan.clustered) cluster.sync();
    if (first.C == 1) {
        if (L < part_len) {
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                o.v[i] = v[i] * P.norm;
                o.idx[i] = P.off + (L - lo) + i;
            }
        }
        return;
    }
    if (first.C == 2) cross_stage<2>(first, buf, o, cluster);
    else if (first.C == 4) cross_stage<4>(first, buf, o, cluster);
    else cross_stage<8>(first, buf, o, cluster);
}

__device__ __forceinline__ void load4_act(const void *x, size_t i, int bf16, float v[4]) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(x) + i);
    const uint32_t w[2] = {raw.x, raw.y};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint16_t bits = (uint16_t)(w[k >> 1] >> (16 * (k & 1)));
        v[k] = bf16 ? __uint_as_float((uint32_t)bits << 16) : __half2float(__ushort_as_half(bits));
    }
}

__global__ void __launch_bounds__(THREADS) rht_in_kernel(RhtInParams p) {
    __shared__ __align__(16) float buf[SEG];
    __shared__ float s_red[THREADS / 32];
    __shared__ long long s_red64[THREADS / 32];
    __shared__ float s_max;      // this part's max |xr| (read by peers)
    __shared__ long long s_sum;  // this part's sum of X (read by peers)
    cg::cluster_group cluster = cg::this_cluster();
    const int part = blockIdx.x, b = blockIdx.y;
    pdl_launch_dependents();
    pdl_wait();  // x comes from the previous kernel on the stream

    const int p0 = p.plan.first_piece[part], p1 = p.plan.first_piece[part + 1];
    int part_len = 0;
    for (int pc = p0; pc < p1; ++pc) part_len += p.plan.piece[pc].len;
    const int L = 4 * threadIdx.x;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    const size_t row = (size_t)b * p.n;
    if (L < part_len) {
        int lo;
        const RhtPiece &P = p.plan.piece[piece_of(p.plan, part, L, lo)];
        const int k0 = P.off + (L - lo);
        load4_act(p.x, row + k0, p.x_bf16, v);
        const uint32_t sw = p.sign_bits[k0 >> 5] >> (k0 & 31);  // 4 aligned bits
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if ((sw >> i) & 1u) v[i] = -v[i];
    }
    Outputs o;
    part_transform(p.plan, part, buf, v, part_len, o, cluster);

    if (p.xr_f32) {  // test entry point: unscaled fp32
#pragma unroll
        for (int r = 0; r < VPT; ++r)
            if (o.idx[r] >= 0) p.xr_f32[row + o.idx[r]] = o.v[r];
        if (p.plan.clustered) cluster.sync();
        return;
    }

    // row max |xr| (each part's max, then all parts in order)
    float mx = 0.f;
#pragma unroll
    for (int r = 0; r < VPT; ++r)
        if (o.idx[r] >= 0) mx = fmaxf(mx, fabsf(o.v[r]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < THREADS / 32; ++w) m = fmaxf(m, s_red[w]);
        s_max = m;
    }
    if (p.plan.clustered) cluster.sync();
    else __syncthreads();
    float rowmax = 0.f;
    for (int q = 0; q < p.plan.parts; ++q)
        rowmax = fmaxf(rowmax, p.plan.clustered ? *cluster.map_shared_rank(&s_max, q) : s_max);
    // X = round(xr 2^e) with rowmax 2^e < 2^14, so |X| <= 16384
    float scale = 1.f;
    if (rowmax > 0.f && isfinite(rowmax)) {
        int e;
        frexpf(rowmax, &e);  // rowmax < 2^e
        scale = ldexpf(1.f, min(14 - e, 126));  // scale and 1 / scale normal for the tiniest rows
    }
    __half *xh = p.xh ? p.xh + (size_t)b * p.n_pad : nullptr;
    if (p.xh_only) {  // tensor-core path: fp16 activations, one rounding
#pragma unroll
        for (int r = 0; r < VPT; ++r)
            if (o.idx[r] >= 0) xh[o.idx[r]] = __float2half_rn(o.v[r] * scale);
        if (part == 0) {
            for (int k = p.n + threadIdx.x; k < p.n_pad; k += THREADS) xh[k] = __float2half(0.f);
            if (threadIdx.x == 0) p.info[b] = glq_rowinfo{0, 1.f / scale, 0.f};
        }
        if (p.plan.clustered) cluster.sync();  // peers may still read this CTA's shared memory
        return;
    }
    uint8_t *xq = p.xq + (size_t)b * p.n_pad * 2;  // per group: 8 high bytes, 8 low bytes
    long long sum = 0;
#pragma unroll
    for (int r = 0; r < VPT; ++r) {
        const int k = o.idx[r];
        if (k >= 0) {
            const int X = __float2int_rn(o.v[r] * scale);
            sum += X;
            const int grp = k >> 3, j = k & 7;
            xq[grp * 16 + j] = (uint8_t)((X >> 8) & 0xFF);
            xq[grp * 16 + 8 + j] = (uint8_t)(X & 0xFF);
            if (xh) xh[k] = __int2half_rn(X);
        }
    }
    if (part == 0) {  // padding columns [n, n_pad) hold zeros
        for (int k = p.n + threadIdx.x; k < p.n_pad; k += THREADS) {
            const int grp = k >> 3, j = k & 7;
            xq[grp * 16 + j] = 0;
            xq[grp * 16 + 8 + j] = 0;
            if (xh) xh[k] = __float2half(0.f);
        }
    }
    // exact row sum of X
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if ((threadIdx.x & 31) == 0) s_red64[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long s = 0;
        for (int w = 0; w < THREADS / 32; ++w) s += s_red64[w];
        s_sum = s;
    }
    if (p.plan.clustered) cluster.sync();
    else __syncthreads();
    if (part == 0 && threadIdx.x == 0) {
        long long total = 0;
        for (int q = 0; q < p.plan.parts; ++q)
            total += p.plan.clustered ? *cluster.map_shared_rank(&s_sum, q) : s_sum;
        p.info[b] = glq_rowinfo{total, 1.f / scale, 0.f};
    }
    if (p.plan.clustered) cluster.sync();  // peers may still read this CTA's shared memory
}

__global__ void __launch_bounds__(THREADS) rht_out_kernel(RhtOutParams p) {
    __shared__ __align__(16) float buf[SEG];
    cg::cluster_group cluster = cg::this_cluster();
    const int part = blockIdx.x, b = blockIdx.y;
    pdl_launch_dependents();
    pdl_wait();  // z comes from the previous kernel

    const int p0 = p.plan.first_piece[part], p1 = p.plan.first_piece[part + 1];
    int part_len = 0;
    for (int pc = p0; pc < p1; ++pc) part_len += p.plan.piece[pc].len;
    const int L = 4 * threadIdx.x;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (L < part_len) {
        int lo;
        const RhtPiece &P = p.plan.piece[piece_of(p.plan, part, L, lo)];
        const int k0 = P.off + (L - lo);
        const float *zr = p.z + (size_t)b * p.z_ld + k0;
        if ((p.z_ld & 3) == 0) {
            const float4 z4 = *reinterpret_cast<const float4 *>(zr);
            v[0] = z4.x; v[1] = z4.y; v[2] = z4.z; v[3] = z4.w;
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = zr[i];
        }
    }
    Outputs o;
    part_transform(p.plan, part, buf, v, part_len, o, cluster);

    const size_t row = (size_t)b * p.m;
#pragma unroll
    for (int r = 0; r < VPT; ++r) {
        const int k = o.idx[r];
        if (k >= 0) {
            const float y = sign_neg(p.sign_bits, k) ? -o.v[r] : o.v[r];
            if (p.y_dtype == 2) {
                reinterpret_cast<float *>(p.y)[row + k] = y;
            } else if (p.y_dtype == 1) {
                reinterpret_cast<__nv_bfloat16 *>(p.y)[row + k] = __float2bfloat16_rn(y);
            } else {
                reinterpret_cast<__half *>(p.y)[row + k] = __float2half_rn(y);
            }
        }
    }
    if (p.plan.clustered) cluster.sync();  // peers may still read this CTA's shared memory
}

template <typename Params>
cudaError_t launch_rht(const void *fn, const Params &p, int B, cudaStream_t s, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.plan.parts, B, 1);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.plan.parts;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    Params q = p;
    void *args[] = {&q};
    return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace

// Plan of a row of length N: blocks of the binary decomposition (descending
// sizes at increasing offsets); blocks above SEG split into C parts whose
// cross stage runs over the cluster, smaller blocks packed whole into parts.
RhtPlan make_rht_plan(int N) {
    RhtPlan plan{};
    int np = 0, parts = 0, off = 0;
    int small_len = SEG + 1;  // length held by the open part of small blocks
    for (int bit = 30; bit >= 0; --bit) {
        if (!(N & (1 << bit))) continue;
        const int K = 1 << bit;
        const float norm = (float)(1.0 / std::sqrt((double)K));
        if (K > SEG) {
            const int C = K / SEG;
            const int rank0 = parts;
            for (int q = 0; q < C; ++q) {
                plan.first_piece[parts++] = np;
                plan.piece[np++] = RhtPiece{off + q * SEG, SEG, K, C, q, rank0, norm};
            }
            small_len = SEG + 1;
        } else {
            if (small_len + K > SEG) {  // open a new part
                plan.first_piece[parts++] = np;
                small_len = 0;
            }
            plan.piece[np++] = RhtPiece{off, K, K, 1, 0, parts - 1, norm};
            small_len += K;
        }
        off += K;
    }
    plan.first_piece[parts] = np;
    plan.parts = parts;
    plan.npieces = np;
    plan.clustered = parts > 1 ? 1 : 0;
    return plan;
}

cudaError_t launch_rht_in(const RhtInParams &p, cudaStream_t s, bool pdl) {
    return launch_rht((const void *)rht_in_kernel, p, p.B, s, pdl);
}

cudaError_t launch_rht_out(const RhtOutParams &p, cudaStream_t s, bool pdl) {
    return launch_rht((const void *)rht_out_kernel, p, p.B, s, pdl);
}

}  // namespace glq
