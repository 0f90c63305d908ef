// mk_inst.cu -- one translation unit per kernel instantiation, compiled once per
// (MK_SPEC, MK_NBT) pair by the build, in parallel: instantiates
// mk_decode_kernel<MK_NBT, MK_SPEC> and exports its host-side launch handle to
// mk_api.cu.
#include "mk_kernel.cuh"

#if !defined(MK_SPEC) || !defined(MK_NBT)
#error "compile with -DMK_SPEC=<0|1|2> -DMK_NBT=<1|2|4|8>"
#endif

#define MK_CAT4(a, b, c, d) a##b##c##d
#define MK_NAME(s, n) MK_CAT4(decode_kernel_s, s, _n, n)

namespace mk {

const void* MK_NAME(MK_SPEC, MK_NBT)() { return (const void*)mk_decode_kernel<MK_NBT, MK_SPEC>; }

}  // namespace mk
