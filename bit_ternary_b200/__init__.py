"""B200-native BitNet b1.58 BitLinear (W1.58-A8): y = F.linear(ActQuant(x), WeightQuant(W)).

The compute path is libbitlinear.so (C ABI, include/bitlinear.h, sm_100a
kernels). `bitlinear` holds the thin PyTorch binding; `workloads` holds the
seeded synthetic inputs. Importing the package does not load the library;
the first call does, and fails loudly if it is missing.
"""
__all__ = ["bitlinear", "workloads", "build"]
