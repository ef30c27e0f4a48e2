"""Leech lattice theta series by the textbook closed form (independent of the oracle).

Theta_Leech = E_12 - (65520/691) * Delta, so the number of vectors of norm 2m is
N(m) = (65520/691) * (sigma_11(m) - tau(m)) for m >= 1 (Conway & Sloane, ch. 2 sec. 2.4 / ch. 4
sec. 11; the pages cite Conway & Sloane and the kissing number 196560).
"""


def tau_coefficients(nmax: int) -> list[int]:
    """Ramanujan tau(1..nmax) from Delta = q * prod_{n>=1} (1 - q^n)^24."""
    poly = [0] * (nmax + 1)
    poly[0] = 1
    for n in range(1, nmax + 1):
        for _ in range(24):
            for d in range(nmax, n - 1, -1):     # multiply by (1 - q^n), in place
                poly[d] -= poly[d - n]
    tau = [0] * (nmax + 1)
    for m in range(1, nmax + 1):
        tau[m] = poly[m - 1]
    return tau


def sigma11(m: int) -> int:
    return sum(d ** 11 for d in range(1, m + 1) if m % d == 0)


def leech_shell_sizes(mmax: int) -> list[int]:
    tau = tau_coefficients(mmax)
    out = [1] + [0] * mmax
    for m in range(1, mmax + 1):
        num = 65520 * (sigma11(m) - tau[m])
        assert num % 691 == 0
        out[m] = num // 691
    return out
