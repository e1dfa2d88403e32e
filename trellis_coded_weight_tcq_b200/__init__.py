"""B200 (sm_100a) trellis-coded quantization: Viterbi encode and bitshift decode.

The compute lives in the CUDA library ``libtcq.so`` (C ABI: ``include/tcq.h``);
``tcq`` is its Python binding and ``workloads`` holds the seeded synthetic
inputs.
"""
from .tcq import (  # noqa: F401
    MAD,
    TCQ_F16,
    TCQ_F32,
    TCQ_MAD,
    Encoded,
    HostPipeline,
    LdlqResult,
    TCQError,
    Workspace,
    bcjr,
    decode,
    decode_vec,
    encode,
    encode_vec,
    gemv,
    gemv_vec,
    ldlq,
    load_library,
    tcq_decode,
    tcq_encode,
    tcq_encode_path,
    tcq_encode_workspace_bytes,
    tcq_gemv,
    tcq_gemv_vec,
    tcq_status_string,
    tcq_words_per_block,
)
