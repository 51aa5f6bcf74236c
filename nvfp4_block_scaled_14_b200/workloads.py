"""Seeded synthetic inputs for the NVFP4 linear layer (shared by the tests, the bench and
the smoke check; holds none of the NVFP4 arithmetic).

Every tensor is drawn on the host from numpy's PCG64 with its own seed,
``seed = 1000 * workload_id + tensor_id``, so the CUDA path and the CPU oracle consume the
same bytes. bf16 tensors are returned as uint16 bit patterns (fp32 draws rounded to nearest
even by torch's CPU cast); FP8 E4M3 tensors as uint8 bit patterns plus their per-tensor scale.

The shapes and distributions stand in for the pages' models (diffusion-transformer hidden
3072 / MLP 12288 at a 64x64 latent, a Qwen3-VL text encoder at decode, and calibration
batches with heavy-tailed entries); the weights, prompts and calibration data themselves are
not available and not needed.
"""
from dataclasses import dataclass, field

import numpy as np
import torch


def rng(workload: int, tensor: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * workload + tensor))


def normal(shape, std, workload, tensor) -> np.ndarray:
    g = rng(workload, tensor)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (torch CPU cast, round to nearest even), as uint16 bit patterns."""
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16) \
        .view(torch.uint16).numpy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def to_fp8_tensorwise(w: np.ndarray):
    """FP8 E4M3 storage with one per-tensor scale (the checkpoint format that double
    quantization starts from): s8 = amax / 448, stored codes = E4M3(w / s8) by torch's
    round-to-nearest-even cast. Returns (uint8 bits, s8)."""
    t = torch.from_numpy(np.ascontiguousarray(w, np.float32))
    s8 = float(t.abs().max()) / 448.0
    s8 = np.float32(s8)
    q = (t / torch.tensor(s8)).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).numpy(), float(s8)


# ---------------------------------------------------------------------------------------
# The five workloads.
# ---------------------------------------------------------------------------------------

@dataclass
class Tiny:
    """fp32 W 256x256 ~ N(0, 0.02^2), X 64x256 ~ N(0, 1); Y = X . W^T (M64 N256 K256)."""
    W: np.ndarray = None
    X: np.ndarray = None
    name: str = "tiny_fp32_m64_n256_k256"


def tiny() -> Tiny:
    return Tiny(W=normal((256, 256), 0.02, 1, 1), X=normal((64, 256), 1.0, 1, 2))


@dataclass
class AttnProj:
    """Double-quant attention projection: W 3072x3072 N(0,0.02^2) stored as FP8 E4M3 with a
    per-tensor scale; X 4096x3072 bf16 N(0,1) with 0.1% of channels (3) scaled x20."""
    W_e4m3: np.ndarray = None
    w_scale: float = 1.0
    X_bf16: np.ndarray = None
    outlier_cols: np.ndarray = None
    name: str = "attn_proj_fp8w_m4096_n3072_k3072"


def attn_proj(M=4096, N=3072, K=3072, workload=2, x_tensor=2) -> AttnProj:
    w = normal((N, K), 0.02, workload, 1)
    w8, s8 = to_fp8_tensorwise(w)
    x = normal((M, K), 1.0, workload, x_tensor)
    n_out = int(round(0.001 * K))
    cols = rng(workload, 3).choice(K, size=max(n_out, 1), replace=False)
    x[:, cols] *= np.float32(20.0)
    return AttnProj(W_e4m3=w8, w_scale=s8, X_bf16=to_bf16_bits(x), outlier_cols=np.sort(cols))


@dataclass
class MlpPair:
    W1: np.ndarray = None  # bf16 bits [12288, 3072]
    W2: np.ndarray = None  # bf16 bits [3072, 12288]
    X1: np.ndarray = None  # bf16 bits [4096, 3072]
    X2: np.ndarray = None  # bf16 bits [4096, 12288], GELU(N(0,1))
    name: str = "dit_mlp_m4096_h3072_f12288"


def mlp_pair(M=4096, H=3072, F=12288, x_tensor=3) -> MlpPair:
    """x_tensor: the seed's tensor id of X1 (X2 takes the next one); other values give other
    activations for the same weights."""
    z = normal((M, F), 1.0, 3, x_tensor + 1)
    x2 = torch.nn.functional.gelu(torch.from_numpy(z)).numpy()
    return MlpPair(W1=to_bf16_bits(normal((F, H), 0.02, 3, 1)),
                   W2=to_bf16_bits(normal((H, F), 0.02, 3, 2)),
                   X1=to_bf16_bits(normal((M, H), 1.0, 3, x_tensor)),
                   X2=to_bf16_bits(x2))


@dataclass
class Decode:
    W: np.ndarray = None  # bf16 bits [12288, 4096]
    X: dict = field(default_factory=dict)  # M -> bf16 bits [M, 4096]
    name: str = "text_encoder_decode_n12288_k4096"


def decode(Ms=(1, 8, 32, 128), N=12288, K=4096) -> Decode:
    d = Decode(W=to_bf16_bits(normal((N, K), 0.015, 4, 1)))
    for i, m in enumerate(Ms):
        d.X[m] = to_bf16_bits(normal((m, K), 1.0, 4, 10 + i))
    return d


def calib_batch(b: int, M=4096, K=3072) -> np.ndarray:
    """Calibration batch b (0..52; 53 is the evaluation batch): N(0,1) with 1% of the
    entries, at seeded positions, replaced by Student-t(3) draws. bf16 bits."""
    g = rng(5, 100 + b)
    x = g.standard_normal(size=(M, K), dtype=np.float32)
    n = x.size
    k = n // 100
    pos = g.choice(n, size=k, replace=False)
    z = g.standard_normal(size=k)
    chi2 = g.chisquare(3, size=k)
    t3 = (z / np.sqrt(chi2 / 3.0)).astype(np.float32)
    x.reshape(-1)[pos] = t3
    return to_bf16_bits(x)


def calib_weight(N=3072, K=3072) -> np.ndarray:
    return to_bf16_bits(normal((N, K), 0.02, 5, 1))


def lowrank_factors(N=3072, K=3072, r=128, std=0.02, workload=2):
    """BF16 low-rank branch of a linear layer (FP4 layers with BF16 rank-128 branches): down
    D [r x K] and up U [N x r], both N(0, std^2), bf16 bits. With x ~ N(0, 1) and K = 3072
    the branch's output has about a fifth of the FP4 product's standard deviation."""
    return (to_bf16_bits(normal((r, K), std, workload, 7)),
            to_bf16_bits(normal((N, r), std, workload, 8)))
