"""Exact rational algebra of irreducible Cartesian tensors, in polynomial form.

Product-side generator (emits the CUDA constants of libflashcart); it never
touches the test reference and the reference never touches it.

Representation: a symmetric rank-l tensor S is held as the homogeneous
polynomial p_S(r) = S . r^{(x)l}, a dict {(px, py, pz): Fraction}.  Entry
S_(px,py,pz) (px x-indices, py y-indices, pz z-indices) is the coefficient
of x^px y^py z^pz divided by the multinomial l!/(px! py! pz!).

Sources (FlashCart, arXiv 2610.06409):
  Sec. 2: STF spaces V_l, admissible paths (l1,l2)->l3, n = (l1+l2-l3)/2.
  Sec. 3: the 2l+1 independent components with p_z <= 1 and the trace
          relation x_{px,py,pz} = -x_{px+2,py,pz-2} - x_{px,py+2,pz-2}.
  App. B: direction tensor T_l and the product Eq. (B1): contract n pairs,
          symmetrise, remove traces; C_{l1l2l3} fixes the normalisation.
  App. C: permutation average x binom(l3, l1-n) = distinct placements.

How each step is written here:
  * contraction of n index pairs of two symmetric tensors = the pairing
    sum_{k1..kn} (d_k1..d_kn p_x)(d_k1..d_kn p_y), scaled by
    (l1-n)!(l2-n)!/(l1! l2!); the polynomial of a tensor is symmetric, so
    this also performs the permutation average;
  * trace removal = harmonic projection of the polynomial,
    h = sum_k (-1)^k (2l-2k-1)!!/((2l-1)!! (2k)!!) |r|^{2k} Laplacian^k p;
  * C_{l1l2l3}: chosen so that (T_l1 (x) T_l2)_l3 = T_l3 (the reading used
    for the normalisation the pages leave to another paper); T_l(z-hat) has
    the polynomial |r|^l P_l(z/|r|) with P_l the Legendre polynomial.
  * odd-J products (App. B, paragraph after Eq. (B1); Sec. 7): one index
    of each input contracted through the Levi-Civita symbol after n pairs,
    then the symmetric trace-free part with no further factor.  In
    polynomial form the epsilon contraction is the triple product
    r . (grad a x grad b) of the n-times paired derivatives a, b, scaled by
    (l1-n-1)!(l2-n-1)!/(l1! l2!).
"""
from fractions import Fraction
from functools import lru_cache
from math import comb, factorial

Poly = dict


def dfact(n):
    f = 1
    while n > 1:
        f *= n
        n -= 2
    return f


def multinomial(l, px, py, pz):
    return factorial(l) // (factorial(px) * factorial(py) * factorial(pz))


# --------------------------------------------------------------------------
# polynomial arithmetic
# --------------------------------------------------------------------------

def p_add(a, b, s=1):
    out = dict(a)
    for m, c in b.items():
        v = out.get(m, 0) + s * c
        if v == 0:
            out.pop(m, None)
        else:
            out[m] = v
    return out


def p_scale(a, s):
    if s == 0:
        return {}
    return {m: c * s for m, c in a.items()}


def p_mul(a, b):
    out = {}
    for ma, ca in a.items():
        for mb, cb in b.items():
            m = (ma[0] + mb[0], ma[1] + mb[1], ma[2] + mb[2])
            v = out.get(m, 0) + ca * cb
            if v == 0:
                out.pop(m, None)
            else:
                out[m] = v
    return out


def p_diff(a, k):
    out = {}
    for m, c in a.items():
        if m[k] == 0:
            continue
        mm = list(m)
        mm[k] -= 1
        out[tuple(mm)] = out.get(tuple(mm), 0) + c * m[k]
    return {m: c for m, c in out.items() if c != 0}


def p_laplacian(a):
    out = {}
    for k in range(3):
        out = p_add(out, p_diff(p_diff(a, k), k))
    return out


R2 = {(2, 0, 0): Fraction(1), (0, 2, 0): Fraction(1), (0, 0, 2): Fraction(1)}


def p_pow(a, n):
    out = {(0, 0, 0): Fraction(1)}
    for _ in range(n):
        out = p_mul(out, a)
    return out


# --------------------------------------------------------------------------
# STF tensors <-> polynomials
# --------------------------------------------------------------------------

def components(l):
    """The 2l+1 independent components (Sec. 3, p_z <= 1), in storage order:
    p_z = 0 with p_x descending, then p_z = 1 with p_x descending."""
    out = [(l - j, j, 0) for j in range(l + 1)]
    out += [(l - 1 - j, j, 1) for j in range(l)]
    return out


def entry_from_components(l, vals, px, py, pz):
    """Entry (px,py,pz) of the STF tensor with independent values `vals`
    (dict component -> Fraction), by the trace relation of Sec. 3."""
    if pz <= 1:
        return vals.get((px, py, pz), Fraction(0))
    return (-entry_from_components(l, vals, px + 2, py, pz - 2)
            - entry_from_components(l, vals, px, py + 2, pz - 2))


def poly_from_components(l, vals):
    out = {}
    for pz in range(l + 1):
        for px in range(l - pz + 1):
            py = l - pz - px
            e = entry_from_components(l, vals, px, py, pz)
            if e != 0:
                out[(px, py, pz)] = e * multinomial(l, px, py, pz)
    return out


def components_from_poly(l, p):
    return [Fraction(p.get(m, 0), multinomial(l, *m)) for m in components(l)]


def harmonic_projection(l, p):
    out = {}
    lap = dict(p)
    r2k = {(0, 0, 0): Fraction(1)}
    for k in range(l // 2 + 1):
        c = Fraction((-1) ** k * dfact(2 * l - 2 * k - 1),
                     dfact(2 * l - 1) * dfact(2 * k))
        out = p_add(out, p_scale(p_mul(r2k, lap), c))
        lap = p_laplacian(lap)
        r2k = p_mul(r2k, R2)
    return out


def contract_pairs(l1, p1, l2, p2, n):
    """polynomial of the n-fold contraction x .n. y (symmetrised)."""
    pairs = [(p1, p2)]
    for _ in range(n):
        nxt = []
        for a, b in pairs:
            for k in range(3):
                da, db = p_diff(a, k), p_diff(b, k)
                if da and db:
                    nxt.append((da, db))
        pairs = nxt
    out = {}
    for a, b in pairs:
        out = p_add(out, p_mul(a, b))
    s = Fraction(factorial(l1 - n) * factorial(l2 - n),
                 factorial(l1) * factorial(l2))
    return p_scale(out, s)


# --------------------------------------------------------------------------
# paths, direction tensors, products
# --------------------------------------------------------------------------

def admissible(l1, l2, l3):
    return abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0


def paths(lin, ledge, lout):
    """Admissible paths ordered by l3, then l1, then l2."""
    return [(l1, l2, l3) for l3 in range(lout + 1) for l1 in range(lin + 1)
            for l2 in range(ledge + 1) if admissible(l1, l2, l3)]


def legendre_coeffs(l):
    """P_l(t) = sum_k a_k t^(l-2k) (Rodrigues / explicit sum)."""
    return [Fraction((-1) ** k * factorial(2 * l - 2 * k),
                     2 ** l * factorial(k) * factorial(l - k) * factorial(l - 2 * k))
            for k in range(l // 2 + 1)]


def direction_zhat_poly(l):
    """Polynomial of T_l(z-hat): |r|^l P_l(z/|r|) = sum_k a_k z^(l-2k) |r|^(2k)."""
    out = {}
    for k, a in enumerate(legendre_coeffs(l)):
        out = p_add(out, p_scale(p_mul({(0, 0, l - 2 * k): Fraction(1)},
                                       p_pow(R2, k)), a))
    return out


def raw_product_poly(l1, p1, l2, p2, l3):
    n = (l1 + l2 - l3) // 2
    q = contract_pairs(l1, p1, l2, p2, n)
    return p_scale(harmonic_projection(l3, q), comb(l3, l1 - n))


@lru_cache(maxsize=None)
def path_norm(l1, l2, l3):
    u = raw_product_poly(l1, direction_zhat_poly(l1), l2,
                         direction_zhat_poly(l2), l3)
    return 1 / u[(0, 0, l3)]


@lru_cache(maxsize=None)
def path_coefficients(l1, l2, l3):
    """K[a][b1][b2] (Fractions): f_a(x, y) = sum K x_b1 y_b2 in independent
    components -- the bilinear polynomial of Sec. 3."""
    n1, n2, n3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    c1, c2 = components(l1), components(l2)
    Cn = path_norm(l1, l2, l3)
    K = [[[Fraction(0)] * n2 for _ in range(n1)] for _ in range(n3)]
    for b1 in range(n1):
        p1 = poly_from_components(l1, {c1[b1]: Fraction(1)})
        for b2 in range(n2):
            p2 = poly_from_components(l2, {c2[b2]: Fraction(1)})
            f = components_from_poly(l3, raw_product_poly(l1, p1, l2, p2, l3))
            for a in range(n3):
                K[a][b1][b2] = f[a] * Cn
    return K


def direction_component_poly(l, comp):
    """Component (px,py,pz) of T_l(u) as a polynomial in u, by counting the
    distinct placements of m identity pairs inside each index letter:
    T_l = (2l-1)!!/l! sum_m (-1)^m (2l-2m-1)!!/(2l-1)!! {u^(l-2m) (x) I^m}."""
    px, py, pz = comp

    def npairs(p, m):
        if 2 * m > p:
            return 0
        return factorial(p) // (factorial(p - 2 * m) * factorial(m) * 2 ** m)
    out = {}
    pre = Fraction(dfact(2 * l - 1), factorial(l))
    for m in range(l // 2 + 1):
        cm = pre * Fraction((-1) ** m * dfact(2 * l - 2 * m - 1), dfact(2 * l - 1))
        for mx in range(m + 1):
            for my in range(m - mx + 1):
                mz = m - mx - my
                cnt = npairs(px, mx) * npairs(py, my) * npairs(pz, mz)
                if cnt == 0:
                    continue
                mono = (px - 2 * mx, py - 2 * my, pz - 2 * mz)
                out[mono] = out.get(mono, 0) + cm * cnt
    return {k: v for k, v in out.items() if v != 0}


def direction_polys(l):
    return [direction_component_poly(l, c) for c in components(l)]


# --------------------------------------------------------------------------
# odd-J (parity-changing) products
# --------------------------------------------------------------------------

def odd_admissible(l1, l2, l3):
    return l1 >= 1 and l2 >= 1 and abs(l1 - l2) <= l3 <= l1 + l2 - 1 and (l1 + l2 + l3) % 2 == 1


def odd_paths(lin, ledge, lout):
    """Odd-J paths ordered by l3, then l1, then l2."""
    return [(l1, l2, l3) for l3 in range(lout + 1) for l1 in range(lin + 1)
            for l2 in range(ledge + 1) if odd_admissible(l1, l2, l3)]


def triple_with_r(a, b):
    """r . (grad a x grad b) as a polynomial."""
    out = {}
    for c in range(3):
        i, j = (c + 1) % 3, (c + 2) % 3
        rc = {tuple(1 if t == c else 0 for t in range(3)): Fraction(1)}
        t = p_add(p_mul(p_diff(a, i), p_diff(b, j)), p_mul(p_diff(a, j), p_diff(b, i)), -1)
        out = p_add(out, p_mul(rc, t))
    return out


def raw_odd_product_poly(l1, p1, l2, p2, l3):
    n = (l1 + l2 - l3 - 1) // 2
    pairs = [(p1, p2)]
    for _ in range(n):
        nxt = []
        for a, b in pairs:
            for k in range(3):
                da, db = p_diff(a, k), p_diff(b, k)
                if da and db:
                    nxt.append((da, db))
        pairs = nxt
    out = {}
    for a, b in pairs:
        out = p_add(out, triple_with_r(a, b))
    s = Fraction(factorial(l1 - n - 1) * factorial(l2 - n - 1), factorial(l1) * factorial(l2))
    return harmonic_projection(l3, p_scale(out, s))


@lru_cache(maxsize=None)
def odd_path_coefficients(l1, l2, l3):
    """K[a][b1][b2] (Fractions) of an odd-J path in independent components."""
    n1, n2, n3 = 2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1
    c1, c2 = components(l1), components(l2)
    K = [[[Fraction(0)] * n2 for _ in range(n1)] for _ in range(n3)]
    for b1 in range(n1):
        p1 = poly_from_components(l1, {c1[b1]: Fraction(1)})
        for b2 in range(n2):
            p2 = poly_from_components(l2, {c2[b2]: Fraction(1)})
            f = components_from_poly(l3, raw_odd_product_poly(l1, p1, l2, p2, l3))
            for a in range(n3):
                K[a][b1][b2] = f[a]
    return K
