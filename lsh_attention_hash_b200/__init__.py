"""B200-native shared-QK LSH attention (Reformer): forward pass and its backward.

The compute path lives in ``liblsh_attention_hash.so`` (hand-written sm_100a
CUDA kernels behind a C ABI declared in ``include/lsh_attention_hash.h``).  This
package is the thin Python binding over that library: argument marshalling
only, with torch used for device memory and streams.  Importing the package
does not load the library; the first call does, and fails loudly if it is
missing.
"""

from .binding import (  # noqa: F401
    LSHError,
    lsh_hash,
    lsh_sort_permute,
    lsh_sort_permute_noalloc,
    lsh_sort_workspace_bytes,
    lsh_chunk_attend,
    lsh_combine_rounds,
    lsh_chunk_attend_backward,
    lsh_get_device_status,
    lsh_attention,
    lsh_attention_host,
    library_path,
    load_library,
)
