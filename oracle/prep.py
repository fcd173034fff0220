"""Operand preparation (oracle): region gather, pooled descriptors, quantisation.

DraftAttention2 abstract and reading note (Method overview, bullets 1 and 4;
Figure 3(b)): queries and keys are reordered into region blocks, pooled per
region (an average descriptor and a channel-wise max descriptor), and
quantised in the same preparation step; V is reordered and transposed as part
of operand packing.

Readings adopted (the pages do not fix them):

* pooling covers a region's real tokens only: the average divides by the
  count of real tokens, the max is the signed maximum per channel;
* INT8 Q/K: one symmetric scale per 64-token block and tensor, from the block's
  absolute maximum over its real tokens and all channels;
* NVFP4 Q/K: microblocks of 16 consecutive channels of one token, e4m3 scale
  from the microblock's absolute maximum / 6, no further outer scale;
* INT8 V: one symmetric scale per channel and head, from the channel's
  absolute maximum over all real tokens of the head;
* NVFP4 V: per channel and head an fp32 outer scale g = amax / (6 * 448); the
  channel is divided by g, then quantised in microblocks of 16 consecutive
  block slots (tokens) with e4m3 scales, so that the microblocks run along the
  reduction axis of P·V;
* padding slots hold zeros (codes 0) and never enter a pooled value.
"""

from __future__ import annotations

import numpy as np

from . import formats as F
from .geometry import block_tokens


def gather_blocks(x_head: np.ndarray, table: np.ndarray):
    """x_head [N, d] → (blocks [nb, S, d] float64 with zero padding, valid [nb, S])."""
    valid = table >= 0
    blocks = np.zeros(table.shape + (x_head.shape[1],), dtype=np.float64)
    blocks[valid] = x_head[table[valid]]
    return blocks, valid


def pool(blocks, valid):
    """(avg [nb, d], max [nb, d]) over each region's real tokens."""
    cnt = valid.sum(1)
    avg = blocks.sum(1) / cnt[:, None]
    masked = np.where(valid[:, :, None], blocks, -np.inf)
    return avg, masked.max(1)


def qk_int8(blocks):
    """INT8 codes [nb, S, d] and fp32 block scales [nb]."""
    amax = np.abs(blocks).max(axis=(1, 2))
    codes, scale = F.int8_quantize(blocks, amax[:, None, None])
    return codes, scale.reshape(-1)


def qk_nvfp4(blocks):
    """e2m1 nibble codes [nb, S, d] and e4m3 scale codes [nb, S, d/16]."""
    return F.nvfp4_quantize(blocks, axis=-1, block=16)


def v_channel_amax(x_head):
    return np.abs(x_head).max(0)


def v_int8(blocks, amax_c):
    """Transposed INT8 V codes [nb, d, S] and fp32 per-channel scales [d]."""
    codes, scale = F.int8_quantize(blocks, amax_c[None, None, :])
    return np.ascontiguousarray(codes.transpose(0, 2, 1)), scale.reshape(-1)


def v_nvfp4(blocks, amax_c):
    """Transposed NVFP4 V: codes [nb, d, S], e4m3 scale codes [nb, d, S/16],
    fp32 outer scale g [d]."""
    g = F.f32_div(amax_c, 6.0 * 448.0)
    nz = g > 0
    r = np.where(nz, F.f32_div(1.0, np.where(nz, g, 1.0)), 0.0)
    vn = F.f32_mul(blocks, r[None, None, :])
    codes, sf = F.nvfp4_quantize(vn, axis=1, block=16)  # microblocks along slots
    return (np.ascontiguousarray(codes.transpose(0, 2, 1)),
            np.ascontiguousarray(sf.transpose(0, 2, 1)), g)


def dequant_v_nvfp4(codes_t, sf_t, g):
    """[nb, d, S] dequantised V (transposed) = g * sf * e2m1."""
    return F.nvfp4_dequantize(codes_t, sf_t, axis=-1, block=16) * g[None, :, None]


def prepare_head(p, q_head, k_head, v_head, table=None):
    """All prepared operands of one (batch, head) as a dict of numpy arrays."""
    if table is None:
        table = block_tokens(p)
    out = {"table": table}
    for name, x in (("q", q_head), ("k", k_head)):
        blocks, valid = gather_blocks(x, table)
        out[name + "_blocks"] = blocks
        out[name + "_avg"], out[name + "_max"] = pool(blocks, valid)
        out[name + "_i8"], out[name + "_s8"] = qk_int8(blocks)
        out[name + "_f4"], out[name + "_sf4"] = qk_nvfp4(blocks)
    vb, valid = gather_blocks(v_head, table)
    out["valid"] = valid
    out["v_blocks"] = vb
    amax_c = v_channel_amax(v_head)
    out["v_i8"], out["v_s8"] = v_int8(vb, amax_c)
    out["v_f4"], out["v_sf4"], out["v_g4"] = v_nvfp4(vb, amax_c)
    return out
