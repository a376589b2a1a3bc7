"""Pins for the metadata encoder of the CPU oracle, and planted mistakes each pin set catches
(CPU only; nothing here runs on a GPU)."""
import types

import numpy as np
import pytest

from oracle import oracle_np as O
from tests import oracle_pins as P

ENCODER_PINS = [P.pin_encoder_golden, P.pin_encoder_exact, P.pin_encoder_agreement, P.pin_snr]


@pytest.mark.parametrize("pin", ENCODER_PINS, ids=lambda p: p.__name__)
def test_encoder_pin(pin):
    pin(O)


def test_encoder_rejects_negative_and_nonfinite():
    with pytest.raises(ValueError):
        O.encode_u8_per_super(np.array([[0.1] * 7 + [-0.1]], np.float32), 8)
    with pytest.raises(ValueError):
        O.encode_i8_per_super(np.array([[0.1] * 15 + [np.inf]], np.float32), 16)


def _enc_unrounded_step(v, per):
    v = np.asarray(v, np.float32)
    N, G = v.shape
    vb = v.reshape(N, G // per, per)
    step = (vb.max(axis=2) / np.float32(255))[..., None]
    codes = np.clip(np.rint(vb / step), 0, 255).astype(np.uint8).reshape(N, G)
    return codes, step[..., 0].astype(np.float16).view(np.uint16)


def _enc_truncating(v, per):
    v = np.asarray(v, np.float32)
    N, G = v.shape
    vb = v.reshape(N, G // per, per)
    s16 = (vb.max(axis=2) / np.float32(255)).astype(np.float16)
    sf = s16.astype(np.float32)[..., None]
    codes = np.clip(np.floor(vb / np.where(sf > 0, sf, 1)), 0, 255).astype(np.uint8).reshape(N, G)
    return codes, s16.view(np.uint16)


def _enc_div256(v, per):
    v = np.asarray(v, np.float32)
    N, G = v.shape
    vb = v.reshape(N, G // per, per)
    s16 = (vb.max(axis=2) / np.float32(256)).astype(np.float16)
    sf = s16.astype(np.float32)[..., None]
    codes = np.clip(np.rint(vb / np.where(sf > 0, sf, 1)), 0, 255).astype(np.uint8).reshape(N, G)
    return codes, s16.view(np.uint16)


def _enc_int6_over_255(v, per):
    v = np.asarray(v, np.float32)
    N, G = v.shape
    vb = v.reshape(N, G // per, per)
    s16 = (np.abs(vb).max(axis=2) / np.float32(255)).astype(np.float16)
    sf = s16.astype(np.float32)[..., None]
    codes = np.clip(np.rint(vb / np.where(sf > 0, sf, 1)), -127, 127).astype(np.int8).reshape(N, G)
    return codes, s16.view(np.uint16)


def _snr_power_ratio(w, w_hat):
    w = np.asarray(w, np.float64)
    e = w - np.asarray(w_hat, np.float64)
    return float(np.log10((w * w).sum() / (e * e).sum()))


MUTANTS = {
    "codes rounded against the unrounded step": dict(encode_u8_per_super=_enc_unrounded_step),
    "codes truncated": dict(encode_u8_per_super=_enc_truncating),
    "step from max / 256": dict(encode_u8_per_super=_enc_div256),
    "int6 step from absmax / 255": dict(encode_i8_per_super=_enc_int6_over_255),
    "snr without the factor 10": dict(snr_db=_snr_power_ratio),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_encoder_mistake_is_caught(name):
    ns = types.SimpleNamespace(**{k: getattr(O, k) for k in dir(O) if not k.startswith("_")})
    for k, v in MUTANTS[name].items():
        setattr(ns, k, v)
    failed = []
    for pin in ENCODER_PINS:
        try:
            pin(ns)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught: {name}"
