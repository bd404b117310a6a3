"""B200-native ISD verify-and-propose step (I-DLM introspective strided decoding).

The compute path is the C-ABI library ``libisd.so`` built from ``csrc/``;
``speculative_verification_isd_b200.isd`` is its Python binding (argument
marshalling only) and raises at import when the library is missing.
``speculative_verification_isd_b200.inputs`` generates seeded synthetic inputs.
"""
__all__ = ["inputs", "isd"]
