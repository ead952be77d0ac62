"""Helpers for the GPU parity tests: seeded inputs on the device and on the host.

The device side gets its packed plane from the library's own pack kernel; the
checker side packs the same trits with its own scalar packer.  Nothing the CUDA
path produces is fed to the checker."""
import numpy as np

import oracle
from ternary_weight_02_b200 import inputs


class Problem:
    """Seeded synthetic ternary linear problem: trits, scales and activations."""

    def __init__(self, M, N, K, fmt, seed=0):
        self.M, self.N, self.K, self.fmt, self.seed = M, N, K, fmt, seed
        # the 1-bit Q1_0 packing holds weights +-1 only
        self.trits = inputs.signs(seed, N, K) if fmt == oracle.FMT_Q1_0 else inputs.trits(seed, N, K)
        self.scales = inputs.scales(seed, N, K, group=oracle.scale_group(fmt))
        self.x = inputs.activations(seed, M, K) if M > 0 else np.zeros((0, K), np.float16)

    # checker side
    def oracle_packed(self):
        return oracle.pack(self.fmt, self.trits)

    def oracle_y(self, apply_hadamard=True):
        return oracle.ternary_linear(self.x, self.oracle_packed(), self.scales, self.N, self.K,
                                     self.fmt, apply_hadamard=apply_hadamard)

    # device side
    def device(self):
        import torch
        from ternary_weight_02_b200 import bonsai as bz
        dev = torch.device("cuda")
        t = torch.from_numpy(self.trits).to(dev)
        packed = bz.pack(self.fmt, t)
        scales = torch.from_numpy(self.scales.view(np.int16)).to(dev).view(torch.float16)
        x = torch.from_numpy(self.x.view(np.int16)).to(dev).view(torch.float16)
        return x, packed, scales


def to_numpy_f16(t):
    return t.detach().cpu().numpy().astype(np.float64)
