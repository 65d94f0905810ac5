"""B200 RNS-CKKS polynomial engine: the data-parallel hot path under encrypted
Transformer inference (NTT, hybrid key switching, rotation, HMult +
relinearisation + rescale, plaintext x ciphertext BSGS products, polynomial
evaluation) as hand-written sm_100a CUDA behind a C ABI (include/he.h).

`he` is the ctypes binding of libhe.so; `torch_io` holds helpers that move
residue arrays between numpy and device tensors.
"""
