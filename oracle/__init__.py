"""CPU oracle (fp64, numpy) for the SRFT-int4 KV-cache path.

TEST INFRASTRUCTURE ONLY: imported by the tests, the package smoke check and
the benchmark's CPU-baseline / reference arm, never by the library.
"""
from .srft_oracle import *  # noqa: F401,F403
from .srft_oracle import (attend_decode, attend_decode_fp16, attend_decode_int4,  # noqa: F401
                          attend_decode_int4_rotated, compressed_bytes_per_vector, decode,
                          dequantize, encode, group_scales,
                          hadamard_matrix, pack_codes, pack_nibbles, qmax, quantize, real_dft_basis, rotation_matrix,
                          srft_forward, srft_inverse, srft_matrix, srht_matrix, unpack_codes,
                          unpack_nibbles)
