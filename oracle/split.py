"""Outlier-channel split (oracle side; test infrastructure).

The pages' fractional bit widths come from splitting a head's channels into
two groups quantized separately: "outlier" channels at a higher bit width,
the "regular" rest at a lower one ("TurboQuant của Google: nén KV cache 6
lần", the correction in the experiments section: 2.5-bit is 32 outlier
channels at 3 bits plus 96 regular channels at 2 bits, >= 4.5x real
compression).  Readings taken here, since the pages give no procedure:

  * each group is its own TurboQuant quantizer on its own sub-vector (its
    own norm, rotation, codebook for its dimension, and for prod its own QJL
    sketch); a group whose size is not a power of two takes the dense (Haar)
    rotation, so both groups here use it;
  * the estimate of <q, x> is the sum of the two groups' estimates; attention
    scores add, and each group's values are summed in its own rotated basis
    and rotated back into its channels;
  * channel selection (the pages name none): the n_o channels with the
    largest mean square over a calibration block of vectors (for a KV cache,
    the first prefill block), ties to the lower index, listed in ascending
    order;
  * the page's own arithmetic for its example is off: (32*3 + 96*2)/128 is
    2.25 bits per channel, not 2.5; the mechanism is the same for any split
    and the average is reported as computed.
"""

from dataclasses import dataclass, field

import numpy as np

from . import quantizer as _qz


def select_outlier_channels(block: np.ndarray, n_o: int) -> np.ndarray:
    """The n_o channels of largest mean square over the rows of ``block``
    ([n, d]), ties to the lower index, in ascending order."""
    ms = np.mean(np.asarray(block, np.float64) ** 2, axis=0)
    order = np.lexsort((np.arange(ms.size), -ms))
    return np.sort(order[:n_o]).astype(np.int64)


@dataclass
class SplitQuantizer:
    d: int
    channels: np.ndarray         # outlier channel indices, ascending
    bits_o: int
    bits_r: int
    variant: str = "mse"
    seed_rot: int = 0
    seed_qjl: int = 1
    outlier: _qz.Quantizer = field(init=False)
    regular: _qz.Quantizer = field(init=False)
    rest: np.ndarray = field(init=False)

    def __post_init__(self):
        ch = np.asarray(self.channels, np.int64)
        assert np.all(np.diff(ch) > 0) and ch.size > 0 and ch[-1] < self.d
        self.channels = ch
        mask = np.ones(self.d, bool)
        mask[ch] = False
        self.rest = np.nonzero(mask)[0]
        self.outlier = _qz.Quantizer(ch.size, self.bits_o, self.variant, seed_rot=self.seed_rot,
                                     seed_qjl=self.seed_qjl, rotation="dense")
        self.regular = _qz.Quantizer(self.rest.size, self.bits_r, self.variant, seed_rot=self.seed_rot + 1,
                                     seed_qjl=self.seed_qjl + 1, rotation="dense")

    @property
    def mean_bits(self) -> float:
        return (self.channels.size * self.bits_o + self.rest.size * self.bits_r) / self.d

    def record_bytes(self) -> int:
        """Stored bytes per vector: both groups' codes, sketches and norms."""
        tot = 0
        for q in (self.outlier, self.regular):
            tot += q.code_bytes + q.qjl_bytes + 4 + (4 if q.prod else 0)
        return tot


def encode(sq: SplitQuantizer, x: np.ndarray, aux: bool = True) -> dict:
    """{"o": encoding of x[:, channels], "r": encoding of the other channels}."""
    x = np.asarray(x, np.float32)
    return {"o": _qz.encode(sq.outlier, np.ascontiguousarray(x[:, sq.channels]), aux=aux),
            "r": _qz.encode(sq.regular, np.ascontiguousarray(x[:, sq.rest]), aux=aux)}


def dequant(sq: SplitQuantizer, enc: dict) -> np.ndarray:
    """Each group's reconstruction put back into its channels (float64)."""
    n = enc["o"]["norms"].shape[0]
    out = np.zeros((n, sq.d))
    out[:, sq.channels] = _qz.dequant(sq.outlier, enc["o"])
    out[:, sq.rest] = _qz.dequant(sq.regular, enc["r"])
    return out


def scores(sq: SplitQuantizer, q: np.ndarray, enc: dict, dtype=np.float64) -> np.ndarray:
    """Estimated <q, x_j> for one query over the records: the two groups'
    asymmetric estimates added."""
    from . import attention as _att
    q = np.asarray(q, dtype)
    return (_att._scores_one(sq.outlier, q[sq.channels], enc["o"], dtype=dtype)
            + _att._scores_one(sq.regular, q[sq.rest], enc["r"], dtype=dtype))


def decode_attention(kq: SplitQuantizer, vq: SplitQuantizer, q: np.ndarray, kenc: dict, venc: dict,
                     scale=None, dtype=np.float64) -> np.ndarray:
    """softmax(<q, k_j> * scale) weighted sum of the values, for one query
    over one (batch, kv head) slice of split-encoded keys and values."""
    from . import attention as _att
    f = dtype
    d = kq.d
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    s = scores(kq, q, kenc, dtype=f)
    logits = s * f(scale)
    e = np.exp(logits - logits.max())
    p = e / e.sum()
    out = np.zeros(d, f)
    out[vq.channels] = _att._values_one(vq.outlier, p, venc["o"], dtype=f)
    out[vq.rest] = _att._values_one(vq.regular, p, venc["r"], dtype=f)
    return out
