"""Seeded attention inputs in the library's layouts (packed grouped-query rows,
K cache [B, Hkv, c_max, hd] in bf16, transposed V cache [B, Hkv, hd, c_max]
holding the bf16 values in fp16) together with the standard layouts the oracle
takes."""

import numpy as np
import torch


def make(B, nq, L0, Hq, Hkv, hd, seed, pad=5):
    rng = np.random.default_rng(seed)
    c_max = (L0 + nq + pad + 7) // 8 * 8
    G = Hq // Hkv
    q = torch.from_numpy(rng.standard_normal((B, nq, Hq, hd)).astype(np.float32)).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((B, Hkv, c_max, hd)).astype(np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, Hkv, c_max, hd)).astype(np.float32)).to(torch.bfloat16)
    v = torch.where(v.abs() < 2.0 ** -14, torch.zeros_like(v), v)  # values fp16 holds exactly
    q_packed = q.reshape(B, nq, Hkv, G, hd).permute(0, 2, 1, 3, 4).contiguous()
    vt = v.transpose(-1, -2).contiguous().to(torch.float16)  # exact: |v| >= 2^-14 or 0
    dev = dict(q=q_packed.cuda(), k=k.cuda(), v=vt.cuda(), c_max=c_max)
    ref = dict(q=q.double().numpy(), k=k.double().numpy().transpose(0, 2, 1, 3)[:, :L0 + nq],
               v=v.double().numpy().transpose(0, 2, 1, 3)[:, :L0 + nq])
    return dev, ref


def bound(ref, n_keys, ref_abs):
    """Per-element error bound of the kernel's bf16 output against the double
    oracle:
      - one bf16 ulp of the output (2^-7 relative: the final rounding plus the
        small error that can push it across a rounding boundary);
      - the probabilities enter the P V product as two fp16 parts, P_hi =
        fp16(P) and P_lo = fp16(P - P_hi) (relative error <= 2^-22 each,
        plus fp16 subnormals of P_lo for the smallest probabilities), so the
        output moves by at most about 2^-22 * (attention over |V|), given as
        ref_abs; 2^-20 leaves a factor 4;
      - an absolute floor for fp32 accumulation in the tensor cores' own
        order: the rounding noise of a sum over n_keys terms grows like
        sqrt(n_keys) * 2^-24 times the size of the partial sums (at most
        max|ref|-sized after normalisation); 2^-22 * sqrt(n_keys) * max|ref|
        leaves a factor 4."""
    return (2.0 ** -7 * np.abs(ref) + 2.0 ** -20 * ref_abs
            + 2.0 ** -22 * np.sqrt(n_keys) * np.abs(ref).max())
