// NCCL entry points resolved at run time.
//
// The sharded engine (mt_create_sharded) is the only user of NCCL. Loading the
// library with dlopen when a sharded context is created, rather than linking
// it, keeps libmt.so free of a load-time NCCL dependency: a process that has
// already loaded an NCCL (PyTorch's, for instance) shares that copy, since
// dlopen of the same soname returns the loaded library, and a process that
// never shards never loads NCCL at all.
#pragma once

#include <nccl.h>

#include <string>

namespace mt {

struct NcclApi {
  ncclResult_t (*GetUniqueId)(ncclUniqueId*) = nullptr;
  ncclResult_t (*CommInitRank)(ncclComm_t*, int, ncclUniqueId, int) = nullptr;
  ncclResult_t (*CommSplit)(ncclComm_t, int, int, ncclComm_t*, ncclConfig_t*) = nullptr;
  ncclResult_t (*CommDestroy)(ncclComm_t) = nullptr;
  ncclResult_t (*AllGather)(const void*, void*, size_t, ncclDataType_t, ncclComm_t, cudaStream_t) = nullptr;
  ncclResult_t (*ReduceScatter)(const void*, void*, size_t, ncclDataType_t, ncclRedOp_t, ncclComm_t,
                                cudaStream_t) = nullptr;
  ncclResult_t (*AllReduce)(const void*, void*, size_t, ncclDataType_t, ncclRedOp_t, ncclComm_t,
                            cudaStream_t) = nullptr;
  const char* (*GetErrorString)(ncclResult_t) = nullptr;
};

// The resolved API, or nullptr with *why set when NCCL cannot be loaded.
const NcclApi* nccl_api(std::string* why);

}  // namespace mt
