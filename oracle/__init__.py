"""CPU oracle of the SVDQuant W4A4 linear layer.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline / reference arm of bench.py, never by the product path.
"""
