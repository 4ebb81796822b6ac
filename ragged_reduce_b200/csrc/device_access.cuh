// Device helpers shared by the register kernels: 16- and 32-byte vector
// loads and stores, and the quotient/remainder ownership arithmetic.
//
// Loads of inputs use the non-coherent path without L1 allocation (inputs
// never overlap outputs within a call; the host checks this); loads of
// small tables read many times (bias, gate rows) keep L1; buffers that a
// call may also write (a residual updated in place, a staging window) use
// plain coherent loads.  Output stores are streaming (.cs).  The 32-byte
// forms are sm_100's 256-bit accesses.
#pragma once

#include <cstdint>

namespace h3rr {

template <int VW>
struct Vec {
    uint32_t r[VW / 4];
};

__device__ __forceinline__ void ld_stream(Vec<16>& v, const char* p)
{
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3])
                 : "l"(p));
}

__device__ __forceinline__ void ld_stream(Vec<32>& v, const char* p)
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3]), "=r"(v.r[4]),
                   "=r"(v.r[5]), "=r"(v.r[6]), "=r"(v.r[7])
                 : "l"(p));
}

__device__ __forceinline__ void ld_cached(Vec<16>& v, const char* p)
{
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3])
                 : "l"(p));
}

__device__ __forceinline__ void ld_cached(Vec<32>& v, const char* p)
{
    asm volatile("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3]), "=r"(v.r[4]),
                   "=r"(v.r[5]), "=r"(v.r[6]), "=r"(v.r[7])
                 : "l"(p));
}

__device__ __forceinline__ void ld_plain(Vec<16>& v, const char* p)
{
    asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3])
                 : "l"(p));
}

__device__ __forceinline__ void ld_plain(Vec<32>& v, const char* p)
{
    asm volatile("ld.global.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v.r[0]), "=r"(v.r[1]), "=r"(v.r[2]), "=r"(v.r[3]), "=r"(v.r[4]),
                   "=r"(v.r[5]), "=r"(v.r[6]), "=r"(v.r[7])
                 : "l"(p));
}

__device__ __forceinline__ void st_stream(char* p, const Vec<16>& v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.r[0]), "r"(v.r[1]),
                 "r"(v.r[2]), "r"(v.r[3])
                 : "memory");
}

__device__ __forceinline__ void st_stream(char* p, const Vec<32>& v)
{
    asm volatile("st.global.cs.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(v.r[0]), "r"(v.r[1]), "r"(v.r[2]), "r"(v.r[3]), "r"(v.r[4]), "r"(v.r[5]),
                 "r"(v.r[6]), "r"(v.r[7])
                 : "memory");
}

__device__ __forceinline__ void st_plain(char* p, const Vec<16>& v)
{
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.r[0]), "r"(v.r[1]),
                 "r"(v.r[2]), "r"(v.r[3])
                 : "memory");
}

__device__ __forceinline__ void st_plain(char* p, const Vec<32>& v)
{
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(v.r[0]), "r"(v.r[1]), "r"(v.r[2]), "r"(v.r[3]), "r"(v.r[4]), "r"(v.r[5]),
                 "r"(v.r[6]), "r"(v.r[7])
                 : "memory");
}

// Owner rank of item x under the quotient/remainder split (q, m) of the
// partition contract, and the first item of rank i.
__device__ __forceinline__ int32_t split_owner(int32_t x, int32_t q, int32_t m)
{
    const int32_t big = m * (q + 1);
    return x < big ? x / (q + 1) : m + (x - big) / q;
}

__device__ __forceinline__ int32_t split_start(int32_t i, int32_t q, int32_t m)
{
    return i * q + (i < m ? i : m);
}

// Token unit v of a launch that covers, for every rank r, the local tokens
// [t0, t0 + cq + (r < cm)) of r's range (a chunk of the token split (tq, tm);
// cq = tq, cm = tm, t0 = 0 for all tokens): the owning rank s, its local
// token tl and the global token t.
struct ChunkToken {
    int32_t s, tl, t;
};

__device__ __forceinline__ ChunkToken chunk_token(int32_t v, int32_t cq, int32_t cm, int32_t t0,
                                                  int32_t tq, int32_t tm)
{
    ChunkToken k;
    k.s = split_owner(v, cq, cm);
    k.tl = t0 + v - split_start(k.s, cq, cm);
    k.t = split_start(k.s, tq, tm) + k.tl;
    return k;
}

}  // namespace h3rr
