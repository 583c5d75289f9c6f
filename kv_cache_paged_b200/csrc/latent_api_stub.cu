// Placeholder until the tcgen05 latent kernel lands.
#include "kvdecode.h"
extern "C" {
size_t kvd_gla_workspace_size(const kvd_gla_params *) { return 0; }
int kvd_gla_decode(const kvd_gla_params *, void *, size_t, kvd_stream_t) { return KVD_ERR_UNSUPPORTED_SHAPE; }
}
