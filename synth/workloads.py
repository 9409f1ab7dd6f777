"""Tensor lists of the synthetic bucket workloads.

Each tensor is (rows, cols, k): a row-major matrix cut into quantisation
blocks of k whole rows (a 1-D tensor of length L is rows=L, cols=1, k=L, i.e.
one block).  Shapes follow the workloads the veScale-FSDP pages evaluate on:
a Llama-style dense layer, a GPT-OSS-style MoE layer, a ragged mix of block
granularities, and a bucket whose gradients live in separate per-tensor
allocations.  Nothing here is optimizer or planner arithmetic.
"""
import math
from dataclasses import dataclass, field
from typing import List

import numpy as np

from .rng import STREAM_SHAPES, stream_key, uniform_f64

# Adam hyper-parameters of every workload (lr, beta1, beta2, eps, weight decay).
HPARAMS = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
PARAM_SIGMA = 0.02      # master weights ~ N(0, 0.02), fp32
GRAD_SIGMA = 1e-3       # gradients ~ N(0, 1e-3), rounded to bf16


@dataclass
class TensorSpec:
    name: str
    rows: int
    cols: int
    k: int
    block_cols: int = 0     # > 0: quantisation tiles of k rows x block_cols columns

    @property
    def numel(self):
        return self.rows * self.cols


@dataclass
class Workload:
    name: str
    tensors: List[TensorSpec]
    m: int                      # simulated ranks (equal slices of the bucket)
    seed: int
    steps: int = 10
    align: int = 16
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def numel(self):
        return sum(t.numel for t in self.tensors)

    def arrays(self):
        """(rows, cols, k) as three int64 numpy arrays in tensor order."""
        r = np.array([t.rows for t in self.tensors], dtype=np.int64)
        c = np.array([t.cols for t in self.tensors], dtype=np.int64)
        k = np.array([t.k for t in self.tensors], dtype=np.int64)
        return r, c, k

    def block_cols(self):
        """Tile widths (0 = whole rows) as an int64 numpy array in tensor order."""
        return np.array([t.block_cols for t in self.tensors], dtype=np.int64)


def _vec(name, n):
    return TensorSpec(name, n, 1, n)


def tiny(m=4):
    """W[512,256] in 16-row blocks, bias[512] and LayerNorm w[256] as single blocks."""
    return Workload("tiny_m4", [TensorSpec("W", 512, 256, 16), _vec("bias", 512), _vec("ln_w", 256)],
                    m=m, seed=0, steps=10,
                    description="W[512,256] k=16, bias[512], LN[256]; m=4; 10 steps")


LLAMA_SHAPES = [("wq", 4096, 4096), ("wk", 1024, 4096), ("wv", 1024, 4096), ("wo", 4096, 4096),
                ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 14336, 4096)]


def _llama_tensors(prefix=""):
    ts = [TensorSpec(prefix + n, r, c, 1) for n, r, c in LLAMA_SHAPES]
    # RMSNorm weights: one row of 4096, block = that row.
    ts += [TensorSpec(prefix + "norm1", 1, 4096, 1), TensorSpec(prefix + "norm2", 1, 4096, 1)]
    return ts


def llama_layer(m=8):
    return Workload("llama_layer_m8", _llama_tensors(), m=m, seed=1, steps=10,
                    description="Llama layer h=4096, GQA 32q/8kv, SwiGLU 14336; 1-row blocks; m=8")


def moe_layer(m=64, experts=32):
    ts = []
    for e in range(experts):
        ts.append(TensorSpec(f"e{e}.gate_up", 5760, 2880, 16))
        ts.append(TensorSpec(f"e{e}.down", 2880, 2880, 16))
    ts.append(TensorSpec("router", 32, 2880, 1))
    ts += [TensorSpec("attn_q", 4096, 2880, 1), TensorSpec("attn_o", 4096, 2880, 1),
           TensorSpec("attn_k", 512, 2880, 1), TensorSpec("attn_v", 512, 2880, 1)]
    name = f"moe_layer_m{m}" if experts == 32 else f"moe_layer_{experts}e_m{m}"
    return Workload(name, ts, m=m, seed=2, steps=10,
                    description=f"MoE layer h=2880, {experts} experts (gate_up 5760x2880, down 2880x2880, "
                                "16-row blocks), router, attention (1-row blocks)")


STRESS_COLS = (1, 1024, 2880, 4096, 7168)
STRESS_KS = (1, 8, 16, 128)


def ragged_stress(m=8, n_tensors=400, target=1_000_000_000, seed=3):
    """400 tensors, rows log-uniform in [64, 16384], cols and k uniform from
    fixed sets, rows rescaled so the bucket holds ~1.0e9 parameters.

    The literal draw averages ~3.5e9 parameters, so rows are multiplied by a
    common factor (iterated until the total is within 0.01% of the target),
    rounded and clamped back to [64, 16384].  k is capped at rows.
    """
    u = uniform_f64(stream_key(seed, STREAM_SHAPES), 0, 3 * n_tensors).reshape(n_tensors, 3)
    lo, hi = math.log(64.0), math.log(16384.0)
    rows0 = np.exp(lo + u[:, 0] * (hi - lo))
    cols = np.array([STRESS_COLS[min(int(x * 5), 4)] for x in u[:, 1]], dtype=np.int64)
    ks = np.array([STRESS_KS[min(int(x * 4), 3)] for x in u[:, 2]], dtype=np.int64)
    f = target / float(np.sum(rows0 * cols))
    rows = None
    for _ in range(50):
        rows = np.clip(np.rint(rows0 * f), 64, 16384).astype(np.int64)
        tot = int(np.sum(rows * cols))
        if abs(tot - target) <= 1e-4 * target:
            break
        f *= target / tot
    ts = [TensorSpec(f"t{i}", int(rows[i]), int(cols[i]), int(min(ks[i], rows[i])))
          for i in range(n_tensors)]
    return Workload(f"ragged_stress_m{m}", ts, m=m, seed=seed, steps=10,
                    description="400 tensors, rows log-uniform [64,16384], cols in "
                                "{1,1024,2880,4096,7168}, k in {1,8,16,128}; ~1.0e9 params")


def copyin(n_tensors=200, m=64):
    """Llama-layer shapes cycled (wq, wk, wv, wo, gate, up, down, norm1, norm2, ...)."""
    base = _llama_tensors()
    ts = []
    for i in range(n_tensors):
        b = base[i % len(base)]
        ts.append(TensorSpec(f"L{i // len(base)}.{b.name}", b.rows, b.cols, b.k))
    return Workload(f"copyin_{n_tensors}_m{m}", ts, m=m, seed=4, steps=20,
                    description=f"Llama-layer shapes cycled to {n_tensors} tensors; grads in "
                                f"{n_tensors} separate allocations; m={m}")


def ragged_mix(m=4, seed=5):
    """Moderate bucket that crosses every code path: per-element blocks,
    8-element blocks, single odd blocks, row blocks below and far above one
    tile, partial last blocks, odd lengths."""
    ts = [
        TensorSpec("vec_b1", 1000, 1, 1),
        TensorSpec("vec_b8", 777, 1, 8),
        _vec("vec_odd", 333),
        TensorSpec("rows48", 300, 48, 16),
        TensorSpec("exp_gu", 129, 2880, 16),
        TensorSpec("big128", 260, 1024, 128),
        TensorSpec("row7168", 5, 7168, 1),
        TensorSpec("odd4099", 1, 4099, 1),
        TensorSpec("b300", 13, 100, 3),
        TensorSpec("small", 2, 3, 1),
        _vec("vec4097", 4097),
        TensorSpec("huge_blk", 40, 7168, 40),
    ]
    return Workload(f"ragged_mix_m{m}", ts, m=m, seed=seed, steps=4,
                    description="ragged mix of block granularities 1..286720 elements")


def llama_layer_tiles(m=8):
    """The Llama layer with 32x32-element quantisation blocks on its matrices
    (32-row layout granularity), RMSNorm weights as one-row blocks."""
    ts = [TensorSpec(n, r, c, 32, 32) for n, r, c in LLAMA_SHAPES]
    ts += [TensorSpec("norm1", 1, 4096, 1), TensorSpec("norm2", 1, 4096, 1)]
    return Workload(f"llama_layer_32x32_m{m}", ts, m=m, seed=1, steps=10,
                    description="Llama layer h=4096 with 32x32 blocks on the matrices; m=8")


def tiles_mix(m=4, seed=6):
    """Moderate bucket over every 2-D block path: several rows per chunk
    (cols <= 4096), one row piece per chunk (cols > 4096) with a narrow last
    strip, 256 tiles in one strip, a tile as wide as a strip, short last row
    blocks, and row-block tensors between them."""
    ts = [
        TensorSpec("t96", 70, 96, 32, 32),
        TensorSpec("t4112", 33, 4112, 32, 64),
        TensorSpec("t1024", 64, 1024, 32, 32),
        TensorSpec("t4096_16", 5, 4096, 2, 16),
        TensorSpec("t8192_wide", 40, 8192, 32, 4096),
        TensorSpec("t48", 48, 48, 16, 16),
        _vec("bias", 300),
        TensorSpec("rows100", 20, 100, 3),
        TensorSpec("t64_k1", 9, 64, 1, 32),
    ]
    return Workload(f"tiles_mix_m{m}", ts, m=m, seed=seed, steps=4,
                    description="2-D block mix: tiles of 16..4096 columns, 1..85 rows per chunk")


_BUILDERS = {
    "tiny_m4": lambda: tiny(4),
    "llama_layer_m8": lambda: llama_layer(8),
    "moe_layer_m64": lambda: moe_layer(64),
    "moe_layer_4e_m64": lambda: moe_layer(64, experts=4),   # profiling-size MoE bucket (1.9 GB moved per step)
    "ragged_stress_m8": lambda: ragged_stress(8),
    "ragged_stress_m128": lambda: ragged_stress(128),
    "ragged_stress_m1024": lambda: ragged_stress(1024),
    "copyin_200_m64": lambda: copyin(200, 64),
    "copyin_9_m64": lambda: copyin(9, 64),
    "ragged_mix_m4": lambda: ragged_mix(4),
    "ragged_mix_m8": lambda: ragged_mix(8),
    "tiles_mix_m4": lambda: tiles_mix(4),
    "tiles_mix_m8": lambda: tiles_mix(8),
    "llama_layer_32x32_m8": lambda: llama_layer_tiles(8),
}
WORKLOAD_NAMES = tuple(_BUILDERS)


def workload(name):
    return _BUILDERS[name]()


# ------------------------------------------------- real-model layer buckets
#
# One FSDP bucket per transformer layer, shapes from the public model
# configurations (recalled; no network to re-check them):
#   DeepSeek-V3: hidden 7168, MLA (q_lora 1536, kv_lora 512, 128 heads, qk
#   nope/rope 128/64, v 128), 256 routed experts + 1 shared (intermediate
#   2048), dense MLP intermediate 18432 in the first 3 layers.
#   GPT-OSS-120B: hidden 2880, 64 query / 8 KV heads of 64, 128 experts with
#   fused gate_up 5760x2880 and down 2880x2880 (with biases), sinks.
# k = rows per quantisation block (1x or 16x row granularity of the pages).

def _k(rows, gran):
    return min(gran, rows)


def deepseek_v3_layer(moe=True, gran=1, m=64):
    H = 7168
    t = []

    def mat(name, r, c):
        t.append(TensorSpec(name, r, c, _k(r, gran)))

    def vec(name, n):
        t.append(_vec(name, n))
    vec("input_layernorm", H)
    mat("q_a_proj", 1536, H)
    vec("q_a_layernorm", 1536)
    mat("q_b_proj", 128 * 192, 1536)
    mat("kv_a_proj_with_mqa", 512 + 64, H)
    vec("kv_a_layernorm", 512)
    mat("kv_b_proj", 128 * 256, 512)
    mat("o_proj", H, 128 * 128)
    vec("post_attention_layernorm", H)
    if moe:
        mat("gate", 256, H)
        vec("e_score_correction_bias", 256)
        for e in range(256):
            mat(f"experts.{e}.gate_proj", 2048, H)
            mat(f"experts.{e}.up_proj", 2048, H)
            mat(f"experts.{e}.down_proj", H, 2048)
        mat("shared.gate_proj", 2048, H)
        mat("shared.up_proj", 2048, H)
        mat("shared.down_proj", H, 2048)
    else:
        mat("mlp.gate_proj", 18432, H)
        mat("mlp.up_proj", 18432, H)
        mat("mlp.down_proj", H, 18432)
    kind = "moe" if moe else "dense"
    return Workload(f"deepseek_v3_{kind}_k{gran}_m{m}", t, m=m, seed=6,
                    description=f"DeepSeek-V3 {kind} layer bucket, {gran}-row blocks")


def gpt_oss_120b_layer(gran=1, m=64):
    H = 2880
    t = []

    def mat(name, r, c):
        t.append(TensorSpec(name, r, c, _k(r, gran)))

    def vec(name, n):
        t.append(_vec(name, n))
    vec("input_layernorm", H)
    mat("q_proj", 64 * 64, H)
    vec("q_proj.bias", 64 * 64)
    mat("k_proj", 8 * 64, H)
    vec("k_proj.bias", 8 * 64)
    mat("v_proj", 8 * 64, H)
    vec("v_proj.bias", 8 * 64)
    mat("o_proj", H, 64 * 64)
    vec("o_proj.bias", H)
    vec("sinks", 64)
    vec("post_attention_layernorm", H)
    mat("router", 128, H)
    vec("router.bias", 128)
    for e in range(128):
        mat(f"experts.{e}.gate_up_proj", 2 * H, H)
        vec(f"experts.{e}.gate_up_proj.bias", 2 * H)
        mat(f"experts.{e}.down_proj", H, H)
        vec(f"experts.{e}.down_proj.bias", H)
    return Workload(f"gpt_oss_120b_k{gran}_m{m}", t, m=m, seed=7,
                    description=f"GPT-OSS-120B layer bucket, {gran}-row blocks")
