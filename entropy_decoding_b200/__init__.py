"""entropy_decoding_b200 -- B200-native (sm_100a) decoding of DFloat11-style
Huffman-coded floating-point exponents.

Modules:
  df11   -- thin ctypes binding of the C-ABI library libdf11.so (encode on
            the host, decode on the GPU); importing it fails loudly when the
            library has not been built.
  synth  -- seeded synthetic weights (no compression arithmetic).
"""
