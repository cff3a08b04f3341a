"""fp64 CPU oracle for SQuad-Attention: test infrastructure, never part of the product path."""
