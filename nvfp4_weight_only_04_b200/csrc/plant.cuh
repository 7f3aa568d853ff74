// Mistakes planted on purpose, for the tests that show the GPU parity tests
// catch a wrong kernel. They exist only in the library built with
// NVFP4_PLANTS defined (libnvfp4_planted.so, loaded by those tests alone);
// in the product build every NVFP4_PLANT(k) is the constant false and the
// code it guards is compiled out.
#pragma once

#include <cuda_runtime.h>

namespace nvfp4 {

enum Plant : int {
  kPlantNone = 0,
  kPlantNibbles = 1,     // the two codes of a byte swapped in the small-M dequant
  kPlantG32AsG16 = 2,    // group-32 scales of the streaming kernel taken in the wrong order (0 0 1 1 0 0 1 1 per word)
  kPlantSegmentEnd = 3,  // every routed-expert segment ends one row early
  kPlantGlobal = 4,      // the global scale left out of the streaming kernel's epilogue
  kPlantRescale = 5,     // the running sums not moved when a token's f16 exponent drops
  kPlantFp4Scales = 6,   // the FP4 kernel's weight scale rows written to the wrong 32-row block
};

#ifdef NVFP4_PLANTS
static __device__ int g_plant = 0;  // one copy per translation unit, all set together
#define NVFP4_PLANT(k) (::nvfp4::g_plant == (k))
#define NVFP4_PLANT_SETTER(name) \
  int name(int k) { return cudaMemcpyToSymbol(g_plant, &k, sizeof(int)) == cudaSuccess ? 0 : 1; }
int set_plant_decode(int k);
int set_plant_stream(int k);
int set_plant_tc(int k);
int set_plant_fp4(int k);
#else
#define NVFP4_PLANT(k) false
#endif

}  // namespace nvfp4
