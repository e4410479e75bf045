// tokn.cu -- instantiations and host launch of the batch-2..8 cluster kernel
// (tokn.cuh), in a translation unit of its own.

#include <mutex>

#include "tokn.cuh"

namespace flint {
namespace {

// Resident 16-CTA clusters of k_tokn<D, I> on the current device (0 if it
// cannot run); cached per device.
template <int D, int I>
int tokn_clusters() {
  auto kern = k_tokn<D, I>;
  static std::mutex mu;
  static int cached[64];
  static bool done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (done[dev]) return cached[dev];
  int n = 0, optin = 0;
  const size_t smem = tn_smem_bytes(D, I);
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
      cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern)) == cudaSuccess &&
      smem + fa.sharedSizeBytes <= static_cast<size_t>(optin) &&
      cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess &&
      cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin - static_cast<int>(fa.sharedSizeBytes)) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kTok1Cluster);
    cfg.blockDim = dim3(kTnWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kTok1Cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kern), &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();  // a refused attribute or query leaves no error behind
  cached[dev] = n;
  done[dev] = true;
  return n;
}

template <int D, int I>
bool tokn_run(int E, int T, bool launch, const TokNParams* t, const TokNMaps* maps, bool pdl, cudaStream_t st,
              cudaError_t* err) {
  if constexpr (!TnShape<D, I>::ok) {
    return false;
  } else {
    if (E > kTnMaxExperts || T < 1 || T > kTnMaxTokens) return false;
    const int nc_max = tokn_clusters<D, I>();
    if (nc_max < 1) return false;
    if (!launch) return true;
    const int nc = std::min(nc_max, T * t->k + t->S);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc * kTok1Cluster);
    cfg.blockDim = dim3(kTnWarps * 32);
    cfg.dynamicSmemBytes = tn_smem_bytes(D, I);
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kTok1Cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    *err = cudaLaunchKernelEx(&cfg, k_tokn<D, I>, *t, *maps);
    return true;
  }
}

template <int D>
bool tokn_d(int I, int E, int T, bool launch, const TokNParams* t, const TokNMaps* maps, bool pdl, cudaStream_t st,
            cudaError_t* err) {
  switch (I) {
    case 256: return tokn_run<D, 256>(E, T, launch, t, maps, pdl, st, err);
    case 512: return tokn_run<D, 512>(E, T, launch, t, maps, pdl, st, err);
    case 1024: return tokn_run<D, 1024>(E, T, launch, t, maps, pdl, st, err);
    default: return false;
  }
}

}  // namespace

bool tokn_dispatch(int d, int I, int E, int T, bool launch, const TokNParams* t, const TokNMaps* maps, bool pdl,
                   cudaStream_t st, cudaError_t* err) {
  switch (d) {
    case 512: return tokn_d<512>(I, E, T, launch, t, maps, pdl, st, err);
    case 1024: return tokn_d<1024>(I, E, T, launch, t, maps, pdl, st, err);
    case 2048: return tokn_d<2048>(I, E, T, launch, t, maps, pdl, st, err);
    default: return false;
  }
}

}  // namespace flint
