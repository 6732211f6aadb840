"""Helpers shared by the GPU parity tests: device buffers, the library handle, oracle comparisons.

Inputs are seeded draws cast to the device dtype on the host (torch CPU), then copied to the
GPU; the oracle receives the same cast values.  Nothing here computes what the method computes.
"""
import numpy as np
import torch

from oracle import spatten_ref as R

BF = torch.bfloat16


def lib():
    from cascade_token_head_b200 import build
    build.build()
    from cascade_token_head_b200 import spatten
    return spatten


def to_dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).cuda()


def host_cast(a, dtype):
    """The float64 values a device tensor of `dtype` holds after a host cast of `a`."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).to(torch.float64).numpy()


def ws(nbytes):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")


def rms(a):
    return float(np.sqrt(np.mean(np.square(np.asarray(a, np.float64))))) + 1e-30


def assert_close_rms(got, ref, frac, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.max(np.abs(got - ref)) if got.size else 0.0
    bound = frac * rms(ref)
    assert err <= bound, f"{what}: max |err| {err:.3e} > {frac} x RMS = {bound:.3e}"
    return err / rms(ref)


def bf16_round_halfwidth(got, ref):
    """Half-width, on the side facing `ref`, of the interval of reals that round to the bf16 value
    `got` (round to nearest even, 8 significant bits): 2**(e-8) for |got| in [2**e, 2**(e+1)),
    except 2**(e-9) below an exact power of two (the binade under it is twice as fine)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    m, x = np.frexp(np.abs(got))                    # |got| = m * 2**x, m in [0.5, 1)
    e = x - 1
    half = np.ldexp(1.0, e - 8)
    toward_zero = np.abs(ref) < np.abs(got)
    half = np.where((m == 0.5) & toward_zero, half / 2, half)
    return np.where(got == 0, 2.0 ** -134, half)


def assert_close_bf16_out(got, ref, frac, what=""):
    """A bf16-stored result must be the bf16 rounding of some value within frac x RMS(ref) of the
    oracle: |got - ref| <= frac x RMS(ref) + the half-width of got's own rounding interval.  This
    is the plain frac x RMS criterion on the computed value, with the storage rounding (at most
    half an ulp of the stored value, and nothing more) taken out."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bound = frac * rms(ref) + bf16_round_halfwidth(got, ref)
    excess = np.abs(got - ref) - bound
    worst = float(excess.max()) if excess.size else -1.0
    assert worst <= 0, f"{what}: error exceeds {frac} x RMS + the bf16 rounding of the stored value by {worst:.3e}"
    return float(np.max(np.abs(got - ref)) / rms(ref)) if got.size else 0.0


def planes_to_host(msb, lsb):
    return msb.cpu().numpy(), lsb.cpu().numpy()


def oracle_quantize_blocks(x32, gain32=None):
    """Oracle quantization of every (b, h) block of x32 [B, H, n, d] (float32 values).
    Returns msb [B,H,n,d] int8, packed lsb [B,H,n,d/2] uint8, scale [B,H] float32."""
    B, H, n, d = x32.shape
    msb = np.empty((B, H, n, d), np.int8)
    lsb = np.empty((B, H, n, d // 2), np.uint8)
    sc = np.empty((B, H), np.float32)
    for b in range(B):
        for h in range(H):
            blk = x32[b, h]
            if gain32 is not None:
                blk = blk * gain32[b][:, None]
            r = R.quantize_head(blk)
            msb[b, h], lsb[b, h], sc[b, h] = r["msb"], R.pack_lsb(r["lsb"]), r["scale"]
    return msb, lsb, sc


def split_heads(x, H, d, which):
    """[B, n, 3*H*d] -> [B, H, n, d] slice of q (0), k (1) or v (2)."""
    B, n, _ = x.shape
    s = x[:, :, which * H * d:(which + 1) * H * d]
    return np.ascontiguousarray(s.reshape(B, n, H, d).transpose(0, 2, 1, 3))
