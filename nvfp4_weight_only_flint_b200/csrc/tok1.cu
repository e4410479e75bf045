// tok1.cu -- instantiations and host launch of the batch-1 cluster kernel
// (tok1.cuh), in a translation unit of its own.

#include <mutex>

#include "tok1.cuh"

namespace flint {
namespace {
// ----------------------------------------------------------------- batch-1 cluster kernel (host)
// Whether the batch-1 cluster kernel serves this shape on the current device:
// its shared memory fits and at least one 16-CTA cluster can be resident.
template <int D, int I, int NE>
bool tok1_ready(int E, size_t* smem_out) {
  auto kern = k_tok1<D, I, NE>;
  static std::mutex mu;
  static int cache_dev[64];
  static int cache_E[64];
  static int cache_ok[64];
  static int n_cache = 0;
  const size_t smem = tok1_smem_bytes(D, I, E);
  *smem_out = smem;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < n_cache; ++i)
    if (cache_dev[i] == dev && cache_E[i] == E) return cache_ok[i] != 0;
  bool ok = false;
  int optin = 0;
  cudaFuncAttributes fa;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess &&
      cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern)) == cudaSuccess &&
      smem + fa.sharedSizeBytes <= static_cast<size_t>(optin) &&
      cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
          cudaSuccess &&
      // the limit is the function's, shared by every E this instantiation
      // serves: the device's whole opt-in budget
      cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize,
                           optin - static_cast<int>(fa.sharedSizeBytes)) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kTok1Cluster);
    cfg.blockDim = dim3(kTok1Warps * 32);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = kTok1Cluster;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    ok = cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void*>(kern), &cfg) == cudaSuccess && n > 0;
  }
  cudaGetLastError();  // a refused attribute or query leaves no sticky error
  if (n_cache < 64) {
    cache_dev[n_cache] = dev;
    cache_E[n_cache] = E;
    cache_ok[n_cache] = ok ? 1 : 0;
    ++n_cache;
  }
  return ok;
}

template <int D, int I, int NE>
cudaError_t launch_tok1_di(const Tok1Params& t, size_t smem, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((t.k + t.S) * kTok1Cluster);
  cfg.blockDim = dim3(kTok1Warps * 32);
  cfg.dynamicSmemBytes = smem;
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
  return cudaLaunchKernelEx(&cfg, k_tok1<D, I, NE>, t);
}

// Dispatch over (d, inter, E class): `ready` checks the shape, else launches.
template <int D, int I>
bool tok1_dispatch_e(int E, bool launch, const Tok1Params* t, bool pdl, cudaStream_t st, cudaError_t* err) {
  size_t smem = 0;
  if (E <= 256) {
    if (!tok1_ready<D, I, 8>(E, &smem)) return false;
    if (launch) *err = launch_tok1_di<D, I, 8>(*t, smem, pdl, st);
  } else {
    if (!tok1_ready<D, I, kMaxExperts / 32>(E, &smem)) return false;
    if (launch) *err = launch_tok1_di<D, I, kMaxExperts / 32>(*t, smem, pdl, st);
  }
  return true;
}

template <int D>
bool tok1_dispatch_i(int I, int E, bool launch, const Tok1Params* t, bool pdl, cudaStream_t st, cudaError_t* err) {
  switch (I) {
    case 128: return tok1_dispatch_e<D, 128>(E, launch, t, pdl, st, err);
    case 256: return tok1_dispatch_e<D, 256>(E, launch, t, pdl, st, err);
    case 512: return tok1_dispatch_e<D, 512>(E, launch, t, pdl, st, err);
    default: return tok1_dispatch_e<D, 1024>(E, launch, t, pdl, st, err);
  }
}

}  // namespace

bool tok1_dispatch(int d, int I, int E, bool launch, const Tok1Params* t, bool pdl, cudaStream_t st,
                   cudaError_t* err) {
  switch (d) {
    case 512: return tok1_dispatch_i<512>(I, E, launch, t, pdl, st, err);
    case 1024: return tok1_dispatch_i<1024>(I, E, launch, t, pdl, st, err);
    case 2048: return tok1_dispatch_i<2048>(I, E, launch, t, pdl, st, err);
    default: return tok1_dispatch_i<4096>(I, E, launch, t, pdl, st, err);
  }
}

}  // namespace flint
