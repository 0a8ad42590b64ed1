"""CPU checks of the identities the long 1D tier relies on (numpy, float64;
no GPU and nothing of the library's device code):

- two real channels in one complex transform: with Z = FFT(u_a + i u_b),
  Y = A Z + D conj(Z(-k)), A = (K_a + K_b)/2, D = (K_a - K_b)/2, gives
  IFFT(Y) = K_a * u_a + i K_b * u_b (both circular convolutions real);
- the split order of a P = P0 P1 (P2) transform: frequency
  k = kap + Po kc (kap the pencil frequency of the levels before the last,
  Po = P / Pc) and its negative -k sit in pencils kap and Po - kap with kc
  reversed (kap != 0) or negated (kap = 0), so the stored half
  kap = 0 .. Po/2 carries every (A, D) by Hermitian symmetry.
(HyenaND pages: arXiv 2607.19378 summary, real-valued kernels on the
zero-padded FFT path; the four-step split is the textbook decomposition.)"""
import numpy as np
import pytest


def _split(n):
    lg = (2 * n).bit_length() - 1
    m = 2 if lg <= 18 else 3
    out, left = [], lg
    for a in range(m):
        share = -(-left // (m - a))
        out.append(1 << share)
        left -= share
    return out


def _pencil(kap, P0, Pm):
    return (kap % P0) * Pm + kap // P0


@pytest.mark.parametrize("P", [64, 256])
def test_two_real_channels_share_one_transform(P):
    rng = np.random.default_rng(P)
    ua, ub, ka, kb = (rng.standard_normal(P) for _ in range(4))
    Ka, Kb = np.fft.fft(ka), np.fft.fft(kb)
    Z = np.fft.fft(ua + 1j * ub)
    Zm = Z[(-np.arange(P)) % P]
    A, D = (Ka + Kb) / 2, (Ka - Kb) / 2
    y = np.fft.ifft(A * Z + D * np.conj(Zm))
    ya = np.real(np.fft.ifft(Ka * np.fft.fft(ua)))
    yb = np.real(np.fft.ifft(Kb * np.fft.fft(ub)))
    assert np.allclose(y.real, ya, atol=1e-12) and np.allclose(y.imag, yb, atol=1e-12)
    # a wrong sign on D or a missing conjugate breaks it
    assert not np.allclose(np.fft.ifft(A * Z - D * np.conj(Zm)).real, ya, atol=1e-6)
    assert not np.allclose(np.fft.ifft(A * Z + D * Zm).real, ya, atol=1e-6)


@pytest.mark.parametrize("n", [512, 1024, 1 << 17, 1 << 18, 1 << 20])
def test_split_order_partner_pencils(n):
    sp = _split(n)
    P = 2 * n
    P0, Pm, Pc = sp[0], (sp[1] if len(sp) == 3 else 1), sp[-1]
    Po = P // Pc
    assert Po * Pc == P
    rng = np.random.default_rng(n % 1000)
    for kap in np.concatenate([[0, 1, Po // 2, Po // 2 - 1, Po // 2 + 1, Po - 1], rng.integers(0, Po, 20)]):
        kap = int(kap)
        for kc in [0, 1, Pc // 2, Pc - 1, int(rng.integers(0, Pc))]:
            k = kap + Po * kc
            mk = (P - k) % P
            kap2, kc2 = mk % Po, mk // Po
            if kap == 0:
                assert kap2 == 0 and kc2 == (Pc - kc) % Pc
            else:
                assert kap2 == Po - kap and kc2 == Pc - 1 - kc
            # the pencil's memory position and back
            o = _pencil(kap, P0, Pm)
            assert 0 <= o < Po and (o // Pm) + P0 * (o % Pm) == kap


def test_stored_half_covers_every_frequency():
    """Every frequency's (A, D) is a stored value or the conjugate of one."""
    n = 1024
    sp = _split(n)
    P, Pc = 2 * n, sp[-1]
    Po = P // Pc
    rng = np.random.default_rng(3)
    Ka = np.fft.fft(rng.standard_normal(P))
    Kb = np.fft.fft(rng.standard_normal(P))
    A, D = (Ka + Kb) / 2, (Ka - Kb) / 2
    stored = {}
    for kap in range(Po // 2 + 1):
        for kc in range(Pc):
            stored[(kap, kc)] = (A[kap + Po * kc], D[kap + Po * kc])
    for k in range(P):
        kap, kc = k % Po, k // Po
        if kap <= Po // 2:
            a, d = stored[(kap, kc)]
        else:
            a, d = (np.conj(x) for x in stored[(Po - kap, Pc - 1 - kc)])
        assert np.isclose(a, A[k]) and np.isclose(d, D[k])
