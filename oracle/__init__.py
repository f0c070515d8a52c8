"""fp64 CPU oracle of the Recurrent Transformer layer (test infrastructure only;
never imported by the product path)."""
